// pkm_noalloc.cu -- pkm_backward_values_noalloc: the sparse value backward with its
// scratch in a fixed device array instead of a caller workspace.
//
// Why it exists: pkm_backward_values needs a workspace of pkm_workspace_size(s, 1)
// bytes, which most callers allocate once. Some callers cannot allocate device
// memory where they run the backward -- for example a serving or training runtime
// that hands out all device memory from its own pool and forbids other
// allocations during its execution phase, or a plugin host that gives the plugin
// device pointers but no allocator. This entry point asks them for nothing beyond
// the inputs and outputs.
//
// The scratch is the file-scope array below. Every GPU that loads this library
// holds it (about 44.2 MiB) until the process exits. Host code only sees a host-side
// stand-in under that name, so the array's device address is looked up with
// cudaGetSymbolAddress, once per device, the first time the entry point runs on
// that device (with that device current).
#include <mutex>

#include "../../include/pkm.h"
#include "pkm_kernels.h"

namespace {

// Limits of the fixed scratch: n*n slots, B*H*k picks and the value width (a bf16 row
// of at most 2048 elements is the widest the kernels take).
constexpr long long kNoAllocMaxSlots = 1LL << 20;  // 1,048,576 slots (n <= 1024)
constexpr long long kNoAllocMaxPicks = 1LL << 21;  // 2,097,152 picks
constexpr int kNoAllocMaxV = 2048;
// The workspace of pkm_backward_values at those limits (its sort buffers, work lists
// and partial rows): about 44.2 MiB.
constexpr size_t kNoAllocBytes = pkm::value_bwd_ws_bytes(kNoAllocMaxPicks, kNoAllocMaxV);

__device__ __align__(256) unsigned char g_pkm_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device; looked up on first use.
int scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PKM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pkm_noalloc_scratch) != cudaSuccess || !p)
      return PKM_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PKM_OK;
}

}  // namespace

extern "C" int pkm_backward_values_noalloc(const pkm_shape* s, const void* values,
                                           const int32_t* indices, const float* weights,
                                           const void* grad_out, float* grad_values,
                                           float* grad_scores, void* stream) {
  if (!s) return PKM_ERR_INVALID_ARG;
  const size_t need = pkm_workspace_size(s, 1);
  if (need == 0) {
    // Invalid shape: let the regular entry point report which error, before any
    // launch (it validates the shape before it looks at the workspace).
    return pkm_backward_values(s, values, indices, weights, grad_out, grad_values, grad_scores,
                               nullptr, 0, stream);
  }
  const long long slots = static_cast<long long>(s->n) * s->n;
  const long long picks = s->B * s->H * static_cast<long long>(s->k);
  if (slots > kNoAllocMaxSlots || picks > kNoAllocMaxPicks || s->v > kNoAllocMaxV ||
      need > kNoAllocBytes)
    return PKM_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != PKM_OK) return rc;
  // The regular entry point zeroes the status word and the work-list lengths on the
  // stream before its kernels use them, and every other part of the scratch is written
  // before it is read, so the previous call's contents do not leak.
  return pkm_backward_values(s, values, indices, weights, grad_out, grad_values, grad_scores,
                             scratch, kNoAllocBytes, stream);
}
