// pkm_tc.h -- tensor-core (tcgen05 / TMEM / TMA) kernels of the query network and
// the per-half sub-key search. Internal interface.
#pragma once

#include <cuda.h>

#include "pkm_kernels.h"

namespace pkm {

// True when the tensor-core kernels take this layer (bf16, tile-aligned sizes).
bool tc_supported(int dtype, int d_model, int H, int dq, int n, int k);

// bf16 planes of q that the scoring kernel reads: hi = RN(q) and lo = RN(q - hi).
constexpr int kScorePlanes = 2;

// q = BN(x W_q^T) written as kScorePlanes bf16 planes [kScorePlanes][B][H*dq]; with
// a.raw_acc, acc = x W_q^T (no BatchNorm) as three planes hi/mid/lo [3][B][H*dq] whose
// sum is the fp32 result to about 2^-24 relative.
cudaError_t launch_query_tc(const LayerArgs& a, void* planes, cudaStream_t st);

// Per-half scores of the q planes against the sub-keys, accumulated in TMEM, and the
// best 32 sub-keys of each half, [B][H][2][32] (in id order, not by score).
cudaError_t launch_score_topk_tc(const LayerArgs& a, const void* planes, float* list_s,
                                 int* list_i, cudaStream_t st);

// Streaming multiprocessors of the current device (cached).
int sm_count();

// bf16 tensor map; dims/strides innermost first, strides in bytes for dims 1..
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B);

// Tensor-core GEMMs of the backward (pkm_gemm_tc.cu). g_planes holds dL/dacc as two
// bf16 planes hi/lo [2][B][F]. grad_x [B][d] = dL/dacc W_q; grad_W [F][d] = dL/dacc^T x.
bool gemm_tc_supported(int64_t B, int F, int d);
cudaError_t launch_grad_x_tc(const void* g_planes, const void* W_q, float* grad_x, int64_t B,
                             int F, int d, int* status, cudaStream_t st);
cudaError_t launch_grad_w_tc(const void* g_planes, const void* x, float* grad_W, int64_t B,
                             int F, int d, int* status, cudaStream_t st);

}  // namespace pkm
