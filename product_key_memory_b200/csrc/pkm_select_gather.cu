// pkm_select_gather.cu -- exact top-k over the k x k product candidates, softmax,
// and the weighted value read summed over heads. Persistent warps, each taking its
// tokens' (token, head) units in order.
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
#include "pkm_tc.h"

namespace pkm {

constexpr int kSgWarps = 4;

// Work units are (token, head) pairs, taken by each warp in token-major order: its
// tokens are t, t + W, t + 2W, ... (W = warps in the grid; the grid is sized to the
// resident blocks, so each warp handles several tokens). A unit's candidate
// selection (warp shuffles, ALU only) would leave the warp without loads in flight,
// so it is software-pipelined: the next unit is selected while the first rows of the
// current unit are in flight, and only a warp's first selection is exposed. The rows
// of a token are still added in pick order (head by head), the heads' rows into one
// fp32 accumulator per lane.
template <typename T, int MAXV>
__global__ void __launch_bounds__(kSgWarps * 32, MAXV >= 8 ? 3 : 4) select_gather_kernel(
    const float* __restrict__ list_s, const int* __restrict__ list_i,
    const T* __restrict__ values, int64_t B, int H, int n, int k, int v,
    float* __restrict__ out, int* __restrict__ indices, float* __restrict__ weights,
    float* __restrict__ scores, int* status) {
  constexpr int VPER = Vec<T>::kPer;
  constexpr int U = MAXV >= 8 ? 1 : 2;  // rows per register buffer (two buffers)
  extern __shared__ int sg_smem[];
  int* pairs = sg_smem;                                  // [kMaxPairs] (a | b << 8)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* rows = sg_smem + kMaxPairs + warp * 4 * kMaxK;    // [2][kMaxK] slots of two units
  float* wts = reinterpret_cast<float*>(rows + 2 * kMaxK);  // [2][kMaxK]
  __shared__ int npairs_s;

  if (threadIdx.x == 0) npairs_s = build_pairs(k, pairs);
  __syncthreads();
  const int npairs = npairs_s;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kSgWarps;
  int64_t t = static_cast<int64_t>(blockIdx.x) * kSgWarps + warp;
  if (t >= B) return;
  const int nvec = v / VPER;

  // Unit (tt, h): exact top-k of the head's candidates, softmax, outputs; its picked
  // slots and weights into rows / wts of `slot` (lanes < k).
  auto select = [&](int64_t tt, int h, int slot) {
    // Per-half lists hold the best 32 sub-keys of each half (in any order; padding has
    // id kIdPad and score -inf). Sorting them puts the best k first.
    const int64_t base = (tt * H + h) * 2 * static_cast<int64_t>(kMaxK);
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
      const int64_t o = (tt * H + h) * static_cast<int64_t>(k) + lane;
      indices[o] = bi;
      weights[o] = w;
      if (scores) scores[o] = bs;
      rows[slot * kMaxK + lane] = bi;
      wts[slot * kMaxK + lane] = w;
    }
  };

  // Weighted value rows: lane covers 16-byte vectors lane, lane+32, ... of each row.
  float acc[MAXV][VPER];
#pragma unroll
  for (int m = 0; m < MAXV; ++m)
#pragma unroll
    for (int e = 0; e < VPER; ++e) acc[m][e] = 0.f;

  auto issue = [&](const int* rr, const float* ww, int r0, uint4 (&raw)[U][MAXV],
                   float (&wr)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      bool live = r0 + u < k;
      int row = live ? rr[r0 + u] : 0;
      if (live && (row < 0 || row >= n * n)) {  // only reachable with NaN scores
        if (lane == 0) record_status(status, kDevBadSlot);
        live = false;
        row = 0;
      }
      wr[u] = live ? ww[r0 + u] : 0.f;
      const T* rp = values + static_cast<int64_t>(row) * v;
#pragma unroll
      for (int m = 0; m < MAXV; ++m) {
        const int vec = lane + 32 * m;
        raw[u][m] = (live && vec < nvec) ? ld_stream_v4(rp + vec * VPER) : make_uint4(0, 0, 0, 0);
      }
    }
  };
  auto accumulate = [&](const uint4 (&raw)[U][MAXV], const float (&wr)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int m = 0; m < MAXV; ++m) {
        float f[VPER];
        Vec<T>::widen(raw[u][m], f);
#pragma unroll
        for (int e = 0; e < VPER; ++e) acc[m][e] = fmaf(wr[u], f[e], acc[m][e]);
      }
  };

  select(t, 0, 0);
  __syncwarp();
  int h = 0, slot = 0;
  for (;;) {
    const int* rr = rows + slot * kMaxK;
    const float* ww = wts + slot * kMaxK;
    uint4 ra[U][MAXV], rb[U][MAXV];
    float wa[U], wb[U];
    issue(rr, ww, 0, ra, wa);
    // The next unit: the next head of this token, else head 0 of the warp's next token.
    int hn = h + 1;
    int64_t tn = t;
    if (hn == H) {
      hn = 0;
      tn = t + stride;
    }
    const bool more = tn < B;  // warp-uniform
    if (more) select(tn, hn, slot ^ 1);
    for (int r0 = 0; r0 < k; r0 += 2 * U) {
      if (r0 + U < k) issue(rr, ww, r0 + U, rb, wb);  // warp-uniform
      accumulate(ra, wa);
      if (r0 + U >= k) break;
      if (r0 + 2 * U < k) issue(rr, ww, r0 + 2 * U, ra, wa);
      accumulate(rb, wb);
    }
    if (hn == 0) {  // token t complete
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
#pragma unroll
        for (int e = 0; e < VPER; ++e) acc[m][e] = 0.f;
      }
    }
    if (!more) break;
    t = tn;
    h = hn;
    slot ^= 1;
    __syncwarp();  // the next unit's rows (written by lanes < k) are visible to all lanes
  }
}

bool select_gather_supported(int H, int k, int v, int dtype) {
  return k >= 1 && k <= kMaxK && H >= 1 && H * k <= 2048 && row_vecs_per_lane(v, dtype) > 0;
}

template <typename T, int MAXV>
static cudaError_t launch_sg(const LayerArgs& a, const float* ls, const int* li, float* out,
                             int* idx, float* w, float* sc, cudaStream_t st) {
  const size_t smem = sizeof(int) * (kMaxPairs + kSgWarps * 4 * kMaxK);
  const void* kern = reinterpret_cast<const void*>(select_gather_kernel<T, MAXV>);
  cudaError_t e = set_max_smem(kern, smem);
  if (e != cudaSuccess) return e;
  // Persistent grid: the blocks that fit on the GPU at once (looked up once per
  // instantiation; the shared-memory size does not limit it), at most one warp per
  // token.
  static int resident = 0;
  if (resident == 0) {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSgWarps * 32, smem);
    if (e != cudaSuccess) return e;
    resident = (per_sm > 0 ? per_sm : 1) * sm_count();
  }
  const int64_t want = (a.B + kSgWarps - 1) / kSgWarps;
  const unsigned grid = static_cast<unsigned>(want < resident ? want : resident);
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
