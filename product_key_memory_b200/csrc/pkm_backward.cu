// pkm_backward.cu -- sparse value backward of the PKM layer.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology: the
// layer is trained end-to-end with sparse updates; Deep Analysis / Methodology:
// every parameter learns by backpropagation while only a few memory slots are
// updated). With L = <grad_out, out> and out = sum_h sum_j w_j V[slot_j]:
//   grad wrt kept score j:  w_j (g_j - sum_l w_l g_l),  g_j = <grad_out[t], V[slot_j]>
//   grad wrt V[slot]:       sum over the picks of that slot of w * grad_out[t]
//
// The value gradient groups the B*H*k picks by slot with a counting sort
// (histogram, exclusive scan, scatter), then one warp walks each window of 32
// sorted picks, sums w * grad_out[t] per slot in registers and writes each slot's
// row once: a plain read-modify-write when the slot's group lies inside the
// window, a vector atomic add only for groups that cross a window edge. Hot slots
// therefore cost one row update per window instead of one per pick.
#include "pkm_common.cuh"
#include "pkm_kernels.h"

namespace pkm {

constexpr int kScanPer = 4;
constexpr int kScanThreads = 1024;
constexpr int kScanBlock = kScanPer * kScanThreads;  // counts per scan block

static int64_t scan_blocks(int64_t slots) { return (slots + kScanBlock - 1) / kScanBlock; }

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t backward_ws_bytes(int64_t B, int H, int k, int64_t slots, BackwardWs* carve, char* base) {
  const int64_t E = B * H * k;
  size_t off = kStatusBytes;
  const size_t o_counts = off;   off += align256(sizeof(int) * slots);
  const size_t o_offsets = off;  off += align256(sizeof(int) * (slots + 1));
  const size_t o_partials = off; off += align256(sizeof(int) * (scan_blocks(slots) + 1));
  const size_t o_order = off;    off += align256(sizeof(int) * (E > 0 ? E : 1));
  if (carve && base) {
    carve->counts = reinterpret_cast<int*>(base + o_counts);
    carve->offsets = reinterpret_cast<int*>(base + o_offsets);
    carve->partials = reinterpret_cast<int*>(base + o_partials);
    carve->order = reinterpret_cast<int*>(base + o_order);
  }
  return off;
}

// ------------------------------------------------------------------ grad_scores
template <typename T, int MAXV>
__global__ void __launch_bounds__(128) grad_scores_kernel(
    const T* __restrict__ values, const T* __restrict__ grad_out,
    const int* __restrict__ indices, const float* __restrict__ weights, int64_t B, int H,
    int k, int v, int64_t slots, float* __restrict__ grad_scores, int* status) {
  constexpr int VPER = Vec<T>::kPer;
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= B) return;
  const int nvec = v / VPER;
  float g[MAXV][VPER];
#pragma unroll
  for (int m = 0; m < MAXV; ++m) {
    const int vec = lane + 32 * m;
    uint4 raw = vec < nvec ? ld_stream_v4(grad_out + t * v + vec * VPER) : make_uint4(0, 0, 0, 0);
    Vec<T>::widen(raw, g[m]);
  }
  for (int h = 0; h < H; ++h) {
    const int64_t base = (t * H + h) * static_cast<int64_t>(k);
    // The head's slot ids, one per lane, handed out by shuffles (no dependent load
    // before each group of row reads).
    const int row_l = lane < k ? indices[base + lane] : 0;
    float gj = 0.f;
    for (int j0 = 0; j0 < k; j0 += U) {
      float part[U];
      uint4 raw[U][MAXV];
      // All U rows' loads are issued before any of them is used.
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const bool live = j0 + u < k;
        int row = __shfl_sync(0xffffffffu, row_l, (j0 + u) & 31);
        const bool ok = live && row >= 0 && row < slots;
        if (live && !ok && lane == 0) record_status(status, kDevBadSlot);
        if (!ok) row = 0;
        const T* rp = values + static_cast<int64_t>(row) * v;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          const int vec = lane + 32 * m;
          raw[u][m] = (ok && vec < nvec) ? ld_stream_v4(rp + vec * VPER) : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        part[u] = 0.f;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          float f[VPER];
          Vec<T>::widen(raw[u][m], f);
#pragma unroll
          for (int e = 0; e < VPER; ++e) part[u] = fmaf(f[e], g[m][e], part[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float s = warp_sum(part[u]);
        if (lane == j0 + u) gj = s;
      }
    }
    const float w = lane < k ? weights[base + lane] : 0.f;
    const float wsum = warp_sum(w * gj);
    if (lane < k && grad_scores) grad_scores[base + lane] = w * (gj - wsum);
  }
}

// --------------------------------------------------------------- counting sort
__global__ void slot_histogram_kernel(const int* __restrict__ indices, int64_t E, int64_t slots,
                                      int* __restrict__ counts, int* status) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < E;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = indices[e];
    if (r >= 0 && r < slots) atomicAdd(counts + r, 1);
    else record_status(status, kDevBadSlot);
  }
}

// Exclusive scan, pass 1: each block scans 4096 counts and emits its total.
__global__ void __launch_bounds__(kScanThreads) scan_local_kernel(
    const int* __restrict__ counts, int64_t slots, int* __restrict__ offsets,
    int* __restrict__ partials) {
  __shared__ int warp_tot[32];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanBlock + threadIdx.x * kScanPer;
  int c[kScanPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    c[i] = base + i < slots ? counts[base + i] : 0;
    sum += c[i];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int wt = warp_tot[lane];
    int wi = wt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - wt;  // exclusive prefix of warp totals
    if (lane == 31) partials[blockIdx.x] = wi;
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - sum;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    if (base + i < slots) offsets[base + i] = run;
    run += c[i];
  }
}

// Pass 2: one block turns the block totals into exclusive block offsets.
__global__ void __launch_bounds__(1024) scan_partials_kernel(int* partials, int64_t nblk) {
  __shared__ int warp_tot[32];
  __shared__ int carry_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int64_t c0 = 0; c0 < nblk; c0 += 1024) {
    const int64_t i = c0 + threadIdx.x;
    const int x = i < nblk ? partials[i] : 0;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wt = warp_tot[lane];
      int wi = wt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      warp_tot[lane] = wi - wt;
    }
    __syncthreads();
    const int carry = carry_s;
    const int excl = carry + warp_tot[warp] + incl - x;
    __syncthreads();
    if (i < nblk) partials[i] = excl;
    if (threadIdx.x == 1023) carry_s = excl + x;
    __syncthreads();
  }
  if (threadIdx.x == 0) partials[nblk] = carry_s;
}

// Pass 3: add each block's offset; the entry past the end holds the total.
__global__ void __launch_bounds__(kScanThreads) scan_add_kernel(int* __restrict__ offsets,
                                                                int64_t slots,
                                                                const int* __restrict__ partials,
                                                                int64_t nblk) {
  const int add = partials[blockIdx.x];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kScanBlock + threadIdx.x * kScanPer;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i)
    if (base + i < slots) offsets[base + i] += add;
  if (blockIdx.x == 0 && threadIdx.x == 0) offsets[slots] = partials[nblk];
}

// Scatter pick ids into their slot's group. Consumes the counts (counts down to 0).
__global__ void slot_scatter_kernel(const int* __restrict__ indices, int64_t E, int64_t slots,
                                    const int* __restrict__ offsets, int* __restrict__ counts,
                                    int* __restrict__ order) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < E;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = indices[e];
    if (r >= 0 && r < slots) {
      const int pos = offsets[r] + atomicSub(counts + r, 1) - 1;
      order[pos] = static_cast<int>(e);
    }
  }
}

// ----------------------------------------------------------- segmented row sums
// One warp per window of 32 sorted picks; total_ptr points at the number of valid
// picks (the last entry of the sort's offsets). Group bounds inside the window come from the
// sorted keys themselves (a ballot on key changes); the keys just before and after
// the window tell whether the first and last groups continue into a neighbour.
template <typename T, int MAXV>
__global__ void __launch_bounds__(128) segment_rows_kernel(
    const int* __restrict__ order, const int* __restrict__ total_ptr,
    const int* __restrict__ indices, const float* __restrict__ weights,
    const T* __restrict__ grad_out, int HK, int v, float* __restrict__ grad_values) {
  constexpr int VPER = Vec<T>::kPer;
  const int lane = threadIdx.x & 31;
  const int total = *total_ptr;
  const int nvec = v / VPER;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t win = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       win * 32 < total; win += nwarps) {
    const int w0 = static_cast<int>(win * 32);
    const int w1 = min(w0 + 32, total);
    int e_l = 0, r_l = -1;
    float wt_l = 0.f;
    if (w0 + lane < w1) {
      e_l = order[w0 + lane];
      r_l = indices[e_l];
      wt_l = weights[e_l];
    }
    // Keys of the picks just outside the window (-1: none).
    int edge = -1;
    if (lane == 0 && w0 > 0) edge = indices[order[w0 - 1]];
    if (lane == 1 && w1 < total) edge = indices[order[w1]];
    const int prev_r = __shfl_sync(0xffffffffu, edge, 0);
    const int next_r = __shfl_sync(0xffffffffu, edge, 1);
    int i = w0;
    while (i < w1) {
      const int r = __shfl_sync(0xffffffffu, r_l, i - w0);
      const unsigned change = __ballot_sync(0xffffffffu, lane > i - w0 && r_l != r);
      const int end = change ? w0 + __ffs(change) - 1 : w1;
      const bool whole = (i > w0 || prev_r != r) && (end < w1 || next_r != r);
      float* grow = grad_values + static_cast<int64_t>(r) * v;
      // A slot group that lies inside this window is owned by this warp: load its row
      // now so the HBM read overlaps the sums below. A group that crosses a window edge
      // is added with vector atomics instead.
      float4 old[MAXV][VPER / 4];
      float acc[MAXV][VPER];
#pragma unroll
      for (int m = 0; m < MAXV; ++m) {
        const int vec = lane + 32 * m;
#pragma unroll
        for (int q = 0; q < VPER; q += 4) {
          old[m][q / 4] = (whole && vec < nvec)
                              ? *reinterpret_cast<const float4*>(grow + vec * VPER + q)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          acc[m][q] = acc[m][q + 1] = acc[m][q + 2] = acc[m][q + 3] = 0.f;
        }
      }
      int j = i;
      for (; j + 1 < end; j += 2) {  // two picks in flight
        const int ea = __shfl_sync(0xffffffffu, e_l, j - w0);
        const int eb = __shfl_sync(0xffffffffu, e_l, j + 1 - w0);
        const float wa = __shfl_sync(0xffffffffu, wt_l, j - w0);
        const float wb = __shfl_sync(0xffffffffu, wt_l, j + 1 - w0);
        const T* ga = grad_out + static_cast<int64_t>(ea / HK) * v;
        const T* gb = grad_out + static_cast<int64_t>(eb / HK) * v;
        uint4 ra[MAXV], rb[MAXV];
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          const int vec = lane + 32 * m;
          ra[m] = vec < nvec ? __ldg(reinterpret_cast<const uint4*>(ga + vec * VPER)) : make_uint4(0, 0, 0, 0);
          rb[m] = vec < nvec ? __ldg(reinterpret_cast<const uint4*>(gb + vec * VPER)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          float fa[VPER], fb[VPER];
          Vec<T>::widen(ra[m], fa);
          Vec<T>::widen(rb[m], fb);
#pragma unroll
          for (int q = 0; q < VPER; ++q) acc[m][q] = fmaf(wb, fb[q], fmaf(wa, fa[q], acc[m][q]));
        }
      }
      if (j < end) {
        const int ea = __shfl_sync(0xffffffffu, e_l, j - w0);
        const float wa = __shfl_sync(0xffffffffu, wt_l, j - w0);
        const T* ga = grad_out + static_cast<int64_t>(ea / HK) * v;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          const int vec = lane + 32 * m;
          if (vec < nvec) {
            float fa[VPER];
            Vec<T>::widen(__ldg(reinterpret_cast<const uint4*>(ga + vec * VPER)), fa);
#pragma unroll
            for (int q = 0; q < VPER; ++q) acc[m][q] = fmaf(wa, fa[q], acc[m][q]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MAXV; ++m) {
        const int vec = lane + 32 * m;
        if (vec < nvec) {
#pragma unroll
          for (int q = 0; q < VPER; q += 4) {
            float4* p = reinterpret_cast<float4*>(grow + vec * VPER + q);
            const float4 o = old[m][q / 4];
            if (whole)
              *p = make_float4(o.x + acc[m][q], o.y + acc[m][q + 1], o.z + acc[m][q + 2],
                               o.w + acc[m][q + 3]);
            else
              atomicAdd(p, make_float4(acc[m][q], acc[m][q + 1], acc[m][q + 2], acc[m][q + 3]));
          }
        }
      }
      i = end;
    }
  }
}

// ------------------------------------------------------------------- launcher
// Stable-enough grouping of E keys in [0, slots): ws.order lists pick ids grouped by
// key, ws.offsets[key] .. ws.offsets[key + 1] is the key's group, ws.offsets[slots]
// the number of valid keys. Keys outside the range are skipped (status word set).
cudaError_t launch_counting_sort(const int* keys, int64_t E, int64_t slots, const BackwardWs& ws,
                                 int* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(ws.counts, 0, sizeof(int) * slots, st);
  if (e != cudaSuccess) return e;
  const int64_t eblocks = (E + 255) / 256;
  const unsigned egrid = static_cast<unsigned>(eblocks < 1 ? 1 : (eblocks < 148 * 32 ? eblocks : 148 * 32));
  slot_histogram_kernel<<<egrid, 256, 0, st>>>(keys, E, slots, ws.counts, status);
  const int64_t nblk = scan_blocks(slots);
  scan_local_kernel<<<static_cast<unsigned>(nblk), kScanThreads, 0, st>>>(ws.counts, slots,
                                                                           ws.offsets, ws.partials);
  scan_partials_kernel<<<1, 1024, 0, st>>>(ws.partials, nblk);
  scan_add_kernel<<<static_cast<unsigned>(nblk), kScanThreads, 0, st>>>(ws.offsets, slots,
                                                                         ws.partials, nblk);
  slot_scatter_kernel<<<egrid, 256, 0, st>>>(keys, E, slots, ws.offsets, ws.counts, ws.order);
  return cudaGetLastError();
}

template <typename T, int MAXV>
static cudaError_t launch_bwd_t(int64_t B, int H, int k, int v, int64_t slots, const void* values,
                                const int* indices, const float* weights, const void* grad_out,
                                float* grad_values, float* grad_scores, const BackwardWs& ws,
                                int* status, cudaStream_t st,
                                const std::function<void()>& between_stages) {
  const int64_t E = B * H * k;
  const T* V = static_cast<const T*>(values);
  const T* G = static_cast<const T*>(grad_out);
  if (grad_scores) {
    const unsigned grid = static_cast<unsigned>((B + 3) / 4);
    grad_scores_kernel<T, MAXV><<<grid, 128, 0, st>>>(V, G, indices, weights, B, H, k, v, slots,
                                                      grad_scores, status);
  }
  between_stages();
  if (!grad_values) return cudaGetLastError();
  cudaError_t e = launch_counting_sort(indices, E, slots, ws, status, st);
  if (e != cudaSuccess) return e;
  const int64_t windows = (E + 31) / 32;
  const int64_t sblocks = (windows + 3) / 4;
  const unsigned sgrid = static_cast<unsigned>(sblocks < 148 * 64 ? sblocks : 148 * 64);
  segment_rows_kernel<T, MAXV><<<sgrid > 0 ? sgrid : 1, 128, 0, st>>>(
      ws.order, ws.offsets + slots, indices, weights, G, H * k, v, grad_values);
  return cudaGetLastError();
}

cudaError_t launch_backward_values(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                                   const void* values, const int* indices, const float* weights,
                                   const void* grad_out, float* grad_values, float* grad_scores,
                                   const BackwardWs& ws, int* status, cudaStream_t st,
                                   const std::function<void()>& between_stages) {
  const int m = row_vecs_per_lane(v, dtype);
#define PKM_BWD(T, M)                                                                        \
  return launch_bwd_t<T, M>(B, H, k, v, slots, values, indices, weights, grad_out, grad_values, \
                            grad_scores, ws, status, st, between_stages)
  if (dtype == 0) {
    switch (m) {
      case 1: PKM_BWD(float, 1);
      case 2: PKM_BWD(float, 2);
      case 4: PKM_BWD(float, 4);
      case 8: PKM_BWD(float, 8);
    }
  } else {
    switch (m) {
      case 1: PKM_BWD(uint16_t, 1);
      case 2: PKM_BWD(uint16_t, 2);
      case 4: PKM_BWD(uint16_t, 4);
      case 8: PKM_BWD(uint16_t, 8);
    }
  }
#undef PKM_BWD
  return cudaErrorInvalidValue;
}

}  // namespace pkm
