// pkm_tc.h -- tensor-core (tcgen05 / TMEM / TMA) kernels of the query network and
// the per-half sub-key search. Internal interface.
#pragma once

#include "pkm_kernels.h"

namespace pkm {

// True when the tensor-core kernels take this layer (bf16, tile-aligned sizes).
bool tc_supported(int dtype, int d_model, int H, int dq, int n, int k);

// q = BN(x W_q^T) written as three bf16 planes hi/mid/lo [3][B][H*dq] whose sum is
// the fp32 result to about 2^-24 relative.
cudaError_t launch_query_tc(const LayerArgs& a, void* planes, cudaStream_t st);

// Per-half scores of the three q planes against the sub-keys, accumulated in TMEM,
// and the best 32 sub-keys of each half, [B][H][2][32] (in id order, not by score).
cudaError_t launch_score_topk_tc(const LayerArgs& a, const void* planes, float* list_s,
                                 int* list_i, cudaStream_t st);

}  // namespace pkm
