// pkm_usage.cu -- memory utilisation of a batch: distinct slots among the picks.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Key Results):
// BatchNorm in the query network raises the share of memory slots in use to over
// 80 %. This counts, for one batch, how many of the n*n slots the B*H*k picks touch:
// one bit per slot, set with atomic OR, then a population count.
#include "pkm_common.cuh"
#include "pkm_kernels.h"

namespace pkm {

__global__ void mark_slots_kernel(const int* __restrict__ indices, int64_t E, int64_t slots,
                                  unsigned* __restrict__ bitmap, int* status) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < E;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = indices[e];
    if (r >= 0 && r < slots) atomicOr(bitmap + (r >> 5), 1u << (r & 31));
    else record_status(status, kDevBadSlot);
  }
}

__global__ void count_bits_kernel(const unsigned* __restrict__ bitmap, int64_t words,
                                  unsigned long long* hits) {
  unsigned long long c = 0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < words;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    c += __popc(bitmap[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0 && c) atomicAdd(hits, c);
}

size_t usage_bitmap_bytes(int64_t slots) { return sizeof(unsigned) * ((slots + 31) / 32); }

cudaError_t launch_slot_usage(const int* indices, int64_t E, int64_t slots, unsigned* bitmap,
                              unsigned long long* hits, int* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(bitmap, 0, usage_bitmap_bytes(slots), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(hits, 0, sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  if (E > 0) {
    const int64_t blocks = (E + 255) / 256;
    mark_slots_kernel<<<static_cast<unsigned>(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, st>>>(
        indices, E, slots, bitmap, status);
  }
  const int64_t words = (slots + 31) / 32;
  const int64_t wblocks = (words + 255) / 256;
  count_bits_kernel<<<static_cast<unsigned>(wblocks < 148 * 4 ? wblocks : 148 * 4), 256, 0, st>>>(
      bitmap, words, hits);
  return cudaGetLastError();
}

}  // namespace pkm
