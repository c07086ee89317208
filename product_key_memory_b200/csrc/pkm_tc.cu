// pkm_tc.cu -- tensor-core kernels (placeholder until the tcgen05 kernels land).
#include "pkm_tc.h"

namespace pkm {

bool tc_supported(int, int, int, int, int, int) { return false; }

cudaError_t launch_query_tc(const LayerArgs&, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_score_topk_tc(const LayerArgs&, const void*, float*, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pkm
