// pkm_select_gather.cu -- exact top-k over the k x k product candidates, softmax,
// and the weighted value read summed over heads. One warp per token.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology and the
// Deep Analysis / Methodology list): the per-half sub-key sets are combined into
// candidate keys, the k keys with the largest inner product are kept, and the
// output is the weighted sum of their value vectors, over the heads. A key's score
// is its left score plus its right score ("Product Keys Give Transformers
// Million-Slot Memory Layers", "Why top-k of each half is enough"); key (i, j) is
// left sub-key i joined with right sub-key j, flat slot i*n + j ("Implied keys vs
// stored sub-keys").
//
// Candidate pruning (pkm_select.cuh): with both per-half lists sorted best first,
// only pairs at list positions (a + 1)(b + 1) <= k can be among the best k -- the
// pages' argument for keeping k per half, applied inside the k x k grid. In fp32 the
// sums keep that order except where two sums round to the same value, which is a
// tie at fp32 resolution.
#include "pkm_common.cuh"
#include "pkm_kernels.h"
#include "pkm_select.cuh"

namespace pkm {

constexpr int kSgWarps = 4;

template <typename T, int MAXV>
__global__ void __launch_bounds__(kSgWarps * 32) select_gather_kernel(
    const float* __restrict__ list_s, const int* __restrict__ list_i,
    const T* __restrict__ values, int64_t B, int H, int n, int k, int v,
    float* __restrict__ out, int* __restrict__ indices, float* __restrict__ weights,
    float* __restrict__ scores, int* status) {
  constexpr int VPER = Vec<T>::kPer;
  constexpr int U = MAXV >= 8 ? 2 : 4;  // rows in flight per lane step
  extern __shared__ int sg_smem[];
  int* pairs = sg_smem;                                  // [kMaxPairs] (a | b << 8)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int HK = H * k;
  int* rows = sg_smem + kMaxPairs + warp * 2 * HK;       // [HK]
  float* wts = reinterpret_cast<float*>(rows + HK);      // [HK]
  __shared__ int npairs_s;

  if (threadIdx.x == 0) npairs_s = build_pairs(k, pairs);
  __syncthreads();
  const int npairs = npairs_s;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kSgWarps + warp;
  if (t >= B) return;

  for (int h = 0; h < H; ++h) {
    // Per-half lists hold the best 32 sub-keys of each half (in any order; padding has
    // id kIdPad and score -inf). Sorting them puts the best k first.
    const int64_t base = (t * H + h) * 2 * static_cast<int64_t>(kMaxK);
    float s1 = list_s[base + lane];
    int i1 = list_i[base + lane];
    float s2 = list_s[base + kMaxK + lane];
    int i2 = list_i[base + kMaxK + lane];
    warp_sort32(s1, i1);
    warp_sort32(s2, i2);
    float bs;
    int bi;
    select_candidates(s1, i1, s2, i2, pairs, npairs, n, bs, bi);
    // Softmax over the k kept scores (lanes 0..k-1 hold them, best first).
    const float mx = __shfl_sync(0xffffffffu, bs, 0);
    const float e = lane < k ? expf(bs - mx) : 0.f;
    const float den = warp_sum(e);
    const float w = e / den;
    if (lane < k) {
      const int64_t o = (t * H + h) * static_cast<int64_t>(k) + lane;
      indices[o] = bi;
      weights[o] = w;
      if (scores) scores[o] = bs;
      rows[h * k + lane] = bi;
      wts[h * k + lane] = w;
    }
  }
  __syncwarp();

  // Weighted value rows: lane covers 16-byte vectors lane, lane+32, ... of each row.
  const int nvec = v / VPER;
  float acc[MAXV][VPER];
#pragma unroll
  for (int m = 0; m < MAXV; ++m)
#pragma unroll
    for (int e = 0; e < VPER; ++e) acc[m][e] = 0.f;

  for (int r0 = 0; r0 < HK; r0 += U) {
    uint4 raw[U][MAXV];
    float wr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      bool live = r0 + u < HK;
      int row = live ? rows[r0 + u] : 0;
      if (live && (row < 0 || row >= n * n)) {  // only reachable with NaN scores
        if (lane == 0) record_status(status, kDevBadSlot);
        live = false;
        row = 0;
      }
      wr[u] = live ? wts[r0 + u] : 0.f;
      const T* rp = values + static_cast<int64_t>(row) * v;
#pragma unroll
      for (int m = 0; m < MAXV; ++m) {
        const int vec = lane + 32 * m;
        raw[u][m] = (live && vec < nvec) ? ld_stream_v4(rp + vec * VPER) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int m = 0; m < MAXV; ++m) {
        float f[VPER];
        Vec<T>::widen(raw[u][m], f);
#pragma unroll
        for (int e = 0; e < VPER; ++e) acc[m][e] = fmaf(wr[u], f[e], acc[m][e]);
      }
  }
  float* orow = out + t * v;
#pragma unroll
  for (int m = 0; m < MAXV; ++m) {
    const int vec = lane + 32 * m;
    if (vec < nvec) {
#pragma unroll
      for (int e = 0; e < VPER; e += 4)
        *reinterpret_cast<float4*>(orow + vec * VPER + e) =
            make_float4(acc[m][e], acc[m][e + 1], acc[m][e + 2], acc[m][e + 3]);
    }
  }
}

bool select_gather_supported(int H, int k, int v, int dtype) {
  return k >= 1 && k <= kMaxK && H >= 1 && H * k <= 2048 && row_vecs_per_lane(v, dtype) > 0;
}

template <typename T, int MAXV>
static cudaError_t launch_sg(const LayerArgs& a, const float* ls, const int* li, float* out,
                             int* idx, float* w, float* sc, cudaStream_t st) {
  const size_t smem = sizeof(int) * (kMaxPairs + kSgWarps * 2 * a.H * a.k);
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(select_gather_kernel<T, MAXV>), smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((a.B + kSgWarps - 1) / kSgWarps);
  select_gather_kernel<T, MAXV><<<grid, kSgWarps * 32, smem, st>>>(
      ls, li, static_cast<const T*>(a.values), a.B, a.H, a.n, a.k, a.v, out, idx, w, sc,
      a.status);
  return cudaGetLastError();
}

cudaError_t launch_select_gather(const LayerArgs& a, const float* ls, const int* li, float* out,
                                 int* idx, float* w, float* sc, cudaStream_t st) {
  const int m = row_vecs_per_lane(a.v, a.dtype);
  if (a.dtype == 0) {
    switch (m) {
      case 1: return launch_sg<float, 1>(a, ls, li, out, idx, w, sc, st);
      case 2: return launch_sg<float, 2>(a, ls, li, out, idx, w, sc, st);
      case 4: return launch_sg<float, 4>(a, ls, li, out, idx, w, sc, st);
      case 8: return launch_sg<float, 8>(a, ls, li, out, idx, w, sc, st);
    }
  } else {
    switch (m) {
      case 1: return launch_sg<uint16_t, 1>(a, ls, li, out, idx, w, sc, st);
      case 2: return launch_sg<uint16_t, 2>(a, ls, li, out, idx, w, sc, st);
      case 4: return launch_sg<uint16_t, 4>(a, ls, li, out, idx, w, sc, st);
      case 8: return launch_sg<uint16_t, 8>(a, ls, li, out, idx, w, sc, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace pkm
