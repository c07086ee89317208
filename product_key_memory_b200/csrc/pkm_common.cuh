// pkm_common.cuh -- device helpers shared by the PKM kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkm {

constexpr int kMaxK = 32;           // keys kept per half / per head handled by a warp
constexpr int kStatusBytes = 256;   // status word region at the head of every workspace
constexpr int kIdPad = 0x7fffffff;  // id of padding entries: loses every tie

// Device status codes written into the workspace status word (first one wins).
enum : int { kDevOk = 0, kDevBadSlot = 1, kDevTimeout = 2, kDevBadShape = 3 };

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ float load_elem(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const uint16_t* p, int64_t i) {
  return __uint_as_float(static_cast<uint32_t>(p[i]) << 16);
}

// 16-byte streaming load that does not allocate in L1 (rows are touched once per token).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Widen one 16-byte vector into fp32 lanes: 8 values for bf16, 4 for fp32.
template <typename T> struct Vec;
template <> struct Vec<uint16_t> {
  static constexpr int kPer = 8;
  __device__ __forceinline__ static void widen(const uint4& r, float* f) {
    f[0] = bf16_lo(r.x); f[1] = bf16_hi(r.x);
    f[2] = bf16_lo(r.y); f[3] = bf16_hi(r.y);
    f[4] = bf16_lo(r.z); f[5] = bf16_hi(r.z);
    f[6] = bf16_lo(r.w); f[7] = bf16_hi(r.w);
  }
};
template <> struct Vec<float> {
  static constexpr int kPer = 4;
  __device__ __forceinline__ static void widen(const uint4& r, float* f) {
    f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
  }
};

// Selection order used by every top-k: higher score first, then lower id.
__device__ __forceinline__ bool better(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// Sort 32 (score, id) pairs held one per lane, best first (bitonic network over shuffles).
__device__ __forceinline__ void warp_sort32(float& s, int& id) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, s, stride);
      const int oi = __shfl_xor_sync(0xffffffffu, id, stride);
      const bool up = (size == 32) || ((lane & size) == 0);
      const bool lower = (lane & stride) == 0;
      const bool keep_better = (lower == up);
      const bool mine_better = better(s, id, os, oi);
      if (keep_better != mine_better) { s = os; id = oi; }
    }
  }
}

// Merge a sorted chunk (cs, ci) into the sorted running list (s, id), keeping the best 32.
// Lane i first takes the better of list[i] and chunk[31 - i] (a bitonic sequence that
// holds the best 32 of the union), then a half-cleaner cascade sorts it.
__device__ __forceinline__ void warp_merge32(float& s, int& id, float cs, int ci) {
  const int lane = threadIdx.x & 31;
  const float rs = __shfl_sync(0xffffffffu, cs, 31 - lane);
  const int ri = __shfl_sync(0xffffffffu, ci, 31 - lane);
  if (better(rs, ri, s, id)) { s = rs; id = ri; }
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const float os = __shfl_xor_sync(0xffffffffu, s, stride);
    const int oi = __shfl_xor_sync(0xffffffffu, id, stride);
    const bool lower = (lane & stride) == 0;
    const bool mine_better = better(s, id, os, oi);
    if (lower != mine_better) { s = os; id = oi; }
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace pkm
