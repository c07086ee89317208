// pkm_util.cu -- host helpers shared by the launchers.
#include <mutex>
#include <vector>

#include "pkm_kernels.h"

namespace pkm {

namespace {
struct SmemSetting {
  const void* func;
  int device;
  size_t bytes;
};
std::mutex g_smem_mu;
std::vector<SmemSetting> g_smem;
}  // namespace

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// (kernel, device, size): cudaFuncSetAttribute is a driver call that otherwise
// costs every launch a few microseconds of host time, which small batches feel.
cudaError_t set_max_smem(const void* func, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_smem_mu);
  for (SmemSetting& s : g_smem)
    if (s.func == func && s.device == dev) {
      if (s.bytes >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(bytes));
      if (e == cudaSuccess) s.bytes = bytes;
      return e;
    }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) g_smem.push_back({func, dev, bytes});
  return e;
}

}  // namespace pkm
