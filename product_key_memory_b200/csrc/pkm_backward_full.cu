// pkm_backward_full.cu -- the rest of the layer's backward: from the kept-score
// gradients into the sub-keys, the query, BatchNorm and the query projection.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology: the
// memory layer is trained end-to-end; Deep Analysis / Methodology: all parameters
// learn by backpropagation). With the picks held fixed (the top-k choice is
// piecewise constant), L = <grad_out, out>, g_c the kept-score gradient, key
// (i, i') = slot (i*n + i'), q = (acc - mean) * s + beta, s = gamma / sqrt(var + eps):
//   dL/dq1 = sum_j g_c[j] C_h[i_j],   dL/dq2 = sum_j g_c[j] C'_h[i'_j]
//   dL/dC_h[i] = sum over picks with i_j = i of g_c q1     (C' likewise with q2)
//   dL/dacc = dL/dq * s,  dL/dgamma = sum_t dL/dq (acc - mean)/sqrt(var + eps),
//   dL/dbeta = sum_t dL/dq,  dL/dW_q = dL/dacc^T x,  dL/dx = dL/dacc W_q.
#include <cuda_bf16.h>

#include "pkm_common.cuh"
#include "pkm_kernels.h"
#include "pkm_tc.h"

namespace pkm {

constexpr int kAccQSmemF = 4096;  // features whose BN scale/shift acc_q_kernel stages

// acc = x W_q^T and q = acc * s + (beta - mean * s), s = gamma / sqrt(var + eps) (the
// forward's query epilogue). With planes, acc = hi + mid + lo from the three bf16 planes
// of the tensor-core query kernel; without, acc is read as is. Eight features per
// thread when F allows it.
__global__ void __launch_bounds__(256) acc_q_kernel(
    const uint16_t* __restrict__ planes, float* __restrict__ acc, float* __restrict__ q,
    const float* __restrict__ mean, const float* __restrict__ var,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps, int B, int F) {
  const int64_t count = static_cast<int64_t>(B) * F;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  extern __shared__ float aq_smem[];  // scale [F], shift [F] when F <= kAccQSmemF
  const bool staged = F <= kAccQSmemF;
  if (staged) {
    for (int f = threadIdx.x; f < F; f += blockDim.x) {
      const float sc = gamma[f] / sqrtf(var[f] + eps);
      aq_smem[f] = sc;
      aq_smem[F + f] = beta[f] - mean[f] * sc;
    }
    __syncthreads();
  }
  if ((F & 7) == 0) {
    const int per_row = F >> 3;
    const int64_t units = static_cast<int64_t>(B) * per_row;
    for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < units;
         u += stride) {
      const int row = static_cast<int>(u / per_row);
      const int f0 = static_cast<int>(u - static_cast<int64_t>(row) * per_row) * 8;
      const int64_t i0 = static_cast<int64_t>(row) * F + f0;
      float a[8];
      if (planes) {
        float h[8], m[8], l[8];
        Vec<uint16_t>::widen(*reinterpret_cast<const uint4*>(planes + i0), h);
        Vec<uint16_t>::widen(*reinterpret_cast<const uint4*>(planes + count + i0), m);
        Vec<uint16_t>::widen(*reinterpret_cast<const uint4*>(planes + 2 * count + i0), l);
#pragma unroll
        for (int j = 0; j < 8; ++j) a[j] = h[j] + m[j] + l[j];
        reinterpret_cast<float4*>(acc + i0)[0] = make_float4(a[0], a[1], a[2], a[3]);
        reinterpret_cast<float4*>(acc + i0)[1] = make_float4(a[4], a[5], a[6], a[7]);
      } else {
        const float4 x = reinterpret_cast<const float4*>(acc + i0)[0];
        const float4 y = reinterpret_cast<const float4*>(acc + i0)[1];
        a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w;
        a[4] = y.x; a[5] = y.y; a[6] = y.z; a[7] = y.w;
      }
      float r[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int f = f0 + j;
        if (staged) {
          r[j] = fmaf(a[j], aq_smem[f], aq_smem[F + f]);
        } else {
          const float sc = gamma[f] / sqrtf(var[f] + eps);
          r[j] = fmaf(a[j], sc, beta[f] - mean[f] * sc);
        }
      }
      reinterpret_cast<float4*>(q + i0)[0] = make_float4(r[0], r[1], r[2], r[3]);
      reinterpret_cast<float4*>(q + i0)[1] = make_float4(r[4], r[5], r[6], r[7]);
    }
    return;
  }
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += stride) {
    float a;
    if (planes) {
      a = load_elem(planes, i) + load_elem(planes, count + i) + load_elem(planes, 2 * count + i);
      acc[i] = a;
    } else {
      a = acc[i];
    }
    const int f = static_cast<int>(i % F);
    const float sc = gamma[f] / sqrtf(var[f] + eps);
    q[i] = fmaf(a, sc, beta[f] - mean[f] * sc);
  }
}

// VW consecutive elements of row r (8 for the vector forms: one 16-byte load of bf16,
// two of fp32).
template <int VW>
__device__ __forceinline__ void load_run(const uint16_t* p, float (&v)[VW]) {
  if constexpr (VW == 8) {
    Vec<uint16_t>::widen(*reinterpret_cast<const uint4*>(p), v);
  } else {
#pragma unroll
    for (int i = 0; i < VW; ++i) v[i] = load_elem(p, i);
  }
}
template <int VW>
__device__ __forceinline__ void load_run(const float* p, float (&v)[VW]) {
  if constexpr (VW == 8) {
    const float4 x = reinterpret_cast<const float4*>(p)[0];
    const float4 y = reinterpret_cast<const float4*>(p)[1];
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
  } else {
#pragma unroll
    for (int i = 0; i < VW; ++i) v[i] = p[i];
  }
}

// VW consecutive fp32 values to p (two 16-byte stores in the vector form; p is then
// 32-byte aligned), optionally added atomically.
template <int VW>
__device__ __forceinline__ void store_run(float* p, const float (&v)[VW], bool atomic) {
  if constexpr (VW == 8) {
    const float4 a = make_float4(v[0], v[1], v[2], v[3]), b = make_float4(v[4], v[5], v[6], v[7]);
    if (atomic) {
      atomicAdd(reinterpret_cast<float4*>(p), a);
      atomicAdd(reinterpret_cast<float4*>(p) + 1, b);
    } else {
      reinterpret_cast<float4*>(p)[0] = a;
      reinterpret_cast<float4*>(p)[1] = b;
    }
  } else {
#pragma unroll
    for (int i = 0; i < VW; ++i) {
      if (atomic) atomicAdd(p + i, v[i]);
      else p[i] = v[i];
    }
  }
}

// One warp per (token, head), lane j holding pick j. For each half the picks that
// share a sub-key are merged: S = sum of their g_c (in pick order), carried by the
// lowest such lane. Then
//   dL/dq_half = sum over distinct sub-keys of S * C_half[sub-key]     (VW per lane)
// and each distinct sub-key becomes one contribution to its gradient row: targets
// [B][H][k][2] (-1 for merged-away picks) with coefficient coef = S.
// dL/dacc = dL/dq * s goes to g_acc (fp32) and/or g_planes (bf16 hi/lo [2][B][F]).
template <typename T, int VW>
__global__ void __launch_bounds__(128) grad_q_targets_kernel(
    const float* __restrict__ g_s, const int* __restrict__ indices, const T* __restrict__ subkeys,
    const float* __restrict__ gamma, const float* __restrict__ var, float eps, int64_t B, int H,
    int dq, int n, int k, float* __restrict__ g_q, float* __restrict__ g_acc,
    uint16_t* __restrict__ g_planes, int* __restrict__ targets, float* __restrict__ coef) {
  const int lane = threadIdx.x & 31;
  const int64_t u = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (u >= B * H) return;
  const int64_t t = u / H;
  const int h = static_cast<int>(u - t * H);
  const int half = dq / 2, F = H * dq;
  const int64_t slots = static_cast<int64_t>(n) * n;
  const int64_t pick = u * k + lane;
  int slot = -1;
  float g = 0.f;
  if (lane < k) {
    slot = indices[pick];
    g = g_s[pick];
  }
  const bool valid = lane < k && slot >= 0 && slot < slots;
  if (!valid) g = 0.f;
  for (int side = 0; side < 2; ++side) {
    // Invalid lanes get distinct negative ids, so they match nobody.
    const int id = valid ? (side ? slot % n : slot / n) : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, id);
    // Every lane of a group runs the same iterations, so the group's mask names exactly
    // the lanes that take part in each shuffle.
    float S = 0.f;
    for (unsigned m = peers; m; m &= m - 1) S += __shfl_sync(peers, g, __ffs(m) - 1);
    const bool leader = valid && (__ffs(peers) - 1 == lane);
    if (lane < k) {
      targets[2 * pick + side] = leader ? (h * 2 + side) * n + id : -1;
      coef[2 * pick + side] = S;
    }
    const unsigned lead = __ballot_sync(0xffffffffu, leader);
    const T* book = subkeys + static_cast<int64_t>(h * 2 + side) * n * half;
    const int f0 = h * dq + side * half;
    for (int e0 = 0; e0 < half; e0 += 32 * VW) {
      const int e = e0 + lane * VW;
      float acc[VW];
#pragma unroll
      for (int i = 0; i < VW; ++i) acc[i] = 0.f;
      // Two distinct rows in flight per step.
      for (unsigned m = lead; m;) {
        const int s0 = __ffs(m) - 1;
        m &= m - 1;
        const int s1 = m ? __ffs(m) - 1 : s0;
        const bool two = m != 0;
        if (two) m &= m - 1;
        const float S0 = __shfl_sync(0xffffffffu, S, s0);
        const int i0 = __shfl_sync(0xffffffffu, id, s0);
        const float S1 = two ? __shfl_sync(0xffffffffu, S, s1) : 0.f;
        const int i1 = __shfl_sync(0xffffffffu, id, s1);
        if (e < half) {
          float r0[VW], r1[VW];
          load_run<VW>(book + static_cast<int64_t>(i0) * half + e, r0);
          load_run<VW>(book + static_cast<int64_t>(i1) * half + e, r1);
#pragma unroll
          for (int i = 0; i < VW; ++i) acc[i] = fmaf(S1, r1[i], fmaf(S0, r0[i], acc[i]));
        }
      }
      if (e < half) {
        const int64_t o = t * F + f0 + e;
        float ga[VW];
        uint16_t ph[VW], pl[VW];
#pragma unroll
        for (int i = 0; i < VW; ++i) {
          const int f = f0 + e + i;
          ga[i] = acc[i] * (gamma[f] / sqrtf(var[f] + eps));
          // hi + lo within 2^-18 relative of ga, for the bf16 GEMMs
          const __nv_bfloat16 hi = __float2bfloat16_rn(ga[i]);
          const __nv_bfloat16 lo = __float2bfloat16_rn(ga[i] - __bfloat162float(hi));
          ph[i] = __bfloat16_as_ushort(hi);
          pl[i] = __bfloat16_as_ushort(lo);
        }
        store_run<VW>(g_q + o, acc, false);
        if (g_acc) store_run<VW>(g_acc + o, ga, false);
        if (g_planes) {
          if constexpr (VW == 8) {
            auto pack = [](const uint16_t (&u)[VW]) {
              return make_uint4(u[0] | (static_cast<uint32_t>(u[1]) << 16),
                                u[2] | (static_cast<uint32_t>(u[3]) << 16),
                                u[4] | (static_cast<uint32_t>(u[5]) << 16),
                                u[6] | (static_cast<uint32_t>(u[7]) << 16));
            };
            *reinterpret_cast<uint4*>(g_planes + o) = pack(ph);
            *reinterpret_cast<uint4*>(g_planes + B * F + o) = pack(pl);
          } else {
#pragma unroll
            for (int i = 0; i < VW; ++i) {
              g_planes[o + i] = ph[i];
              g_planes[B * F + o + i] = pl[i];
            }
          }
        }
      }
    }
  }
}

// Column sums over tokens, pass 1: block (feature group of 256, token chunk) writes its
// partial dL/dbeta and dL/dgamma sums; pass 2 adds the chunks in a fixed order.
constexpr int kBnChunks = 128;

__global__ void bn_grad_partial_kernel(const float* __restrict__ g_q, const float* __restrict__ acc,
                                       const float* __restrict__ mean,
                                       const float* __restrict__ var, float eps, int64_t B, int F,
                                       float* __restrict__ part) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= F) return;
  const int64_t per = (B + kBnChunks - 1) / kBnChunks;
  const int64_t t0 = blockIdx.y * per, t1 = min(B, t0 + per);
  const float mu = mean[f], rs = 1.f / sqrtf(var[f] + eps);
  float sb = 0.f, sg = 0.f;
#pragma unroll 4
  for (int64_t t = t0; t < t1; ++t) {
    const float g = g_q[t * F + f];
    sb += g;
    sg = fmaf(g, (acc[t * F + f] - mu) * rs, sg);
  }
  part[static_cast<int64_t>(blockIdx.y) * 2 * F + f] = sb;
  part[static_cast<int64_t>(blockIdx.y) * 2 * F + F + f] = sg;
}

// Pass 2: block = 32 features x 8 warps; warp w adds chunks [16 w, 16 w + 16) in
// order, then warp 0 adds the 8 warp sums in order (a fixed order: deterministic).
constexpr int kBnFinalWarps = 8;
static_assert(kBnChunks % kBnFinalWarps == 0, "chunks split evenly over the warps");

__global__ void __launch_bounds__(kBnFinalWarps * 32) bn_grad_final_kernel(
    const float* __restrict__ part, int F, float* __restrict__ grad_gamma,
    float* __restrict__ grad_beta, float* __restrict__ sums) {
  __shared__ float wb[kBnFinalWarps][32], wg[kBnFinalWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * 32 + lane;
  constexpr int per = kBnChunks / kBnFinalWarps;
  float pb = 0.f, pg = 0.f;
  if (f < F) {
#pragma unroll 4
    for (int c = warp * per; c < (warp + 1) * per; ++c) {
      pb += part[static_cast<int64_t>(c) * 2 * F + f];
      pg += part[static_cast<int64_t>(c) * 2 * F + F + f];
    }
  }
  wb[warp][lane] = pb;
  wg[warp][lane] = pg;
  __syncthreads();
  if (warp != 0 || f >= F) return;
  float sb = 0.f, sg = 0.f;
#pragma unroll
  for (int w = 0; w < kBnFinalWarps; ++w) {
    sb += wb[w][lane];
    sg += wg[w][lane];
  }
  if (grad_beta) grad_beta[f] = sb;
  if (grad_gamma) grad_gamma[f] = sg;
  if (sums) {
    sums[f] = sb;
    sums[F + f] = sg;
  }
}

// Sub-key gradient rows from the contributions grouped by target: one warp per window
// of 32 sorted contributions, a contribution c adding coef[c] * q_half[token] to its
// row (VW elements per lane, two contributions in flight). Groups inside a window are
// written once (the table was zeroed); groups crossing a window edge add atomically.
template <int VW>
__global__ void __launch_bounds__(128) segment_subkeys_kernel(
    const int* __restrict__ order, const int* __restrict__ total_ptr,
    const int* __restrict__ targets, const float* __restrict__ coef,
    const float* __restrict__ q, int H, int dq, int n, int k,
    float* __restrict__ grad_subkeys) {
  const int lane = threadIdx.x & 31;
  const int total = *total_ptr;
  const int half = dq / 2, F = H * dq, HK = H * k;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t win = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       win * 32 < total; win += nwarps) {
    const int w0 = static_cast<int>(win * 32);
    const int w1 = min(w0 + 32, total);
    int tg_l = -1, t_l = 0;
    float cf_l = 0.f;
    if (w0 + lane < w1) {
      const int c = order[w0 + lane];
      tg_l = targets[c];
      cf_l = coef[c];
      t_l = (c >> 1) / HK;
    }
    // Group bounds from the sorted keys; the keys just outside the window tell
    // whether the first and last groups continue into a neighbour (-1: none).
    int edge = -1;
    if (lane == 0 && w0 > 0) edge = targets[order[w0 - 1]];
    if (lane == 1 && w1 < total) edge = targets[order[w1]];
    const int prev_t = __shfl_sync(0xffffffffu, edge, 0);
    const int next_t = __shfl_sync(0xffffffffu, edge, 1);
    int i = w0;
    while (i < w1) {
      const int tg = __shfl_sync(0xffffffffu, tg_l, i - w0);
      const unsigned change = __ballot_sync(0xffffffffu, lane > i - w0 && tg_l != tg);
      const int end = change ? w0 + __ffs(change) - 1 : w1;
      const bool whole = (i > w0 || prev_t != tg) && (end < w1 || next_t != tg);
      const int side = (tg / n) & 1;
      const int h = tg / (2 * n);
      const float* qbase = q + h * dq + side * half;
      float* grow = grad_subkeys + static_cast<int64_t>(tg) * half;
      for (int e0 = 0; e0 < half; e0 += 32 * VW) {
        const int e = e0 + lane * VW;
        const bool in = e < half;
        float sum[VW];
#pragma unroll
        for (int m = 0; m < VW; ++m) sum[m] = 0.f;
        int j = i;
        for (; j + 1 < end; j += 2) {
          const float ca = __shfl_sync(0xffffffffu, cf_l, j - w0);
          const int ta = __shfl_sync(0xffffffffu, t_l, j - w0);
          const float cb = __shfl_sync(0xffffffffu, cf_l, j + 1 - w0);
          const int tb = __shfl_sync(0xffffffffu, t_l, j + 1 - w0);
          if (in) {
            float ra[VW], rb[VW];
            load_run<VW>(qbase + static_cast<int64_t>(ta) * F + e, ra);
            load_run<VW>(qbase + static_cast<int64_t>(tb) * F + e, rb);
#pragma unroll
            for (int m = 0; m < VW; ++m) sum[m] = fmaf(cb, rb[m], fmaf(ca, ra[m], sum[m]));
          }
        }
        if (j < end) {
          const float ca = __shfl_sync(0xffffffffu, cf_l, j - w0);
          const int ta = __shfl_sync(0xffffffffu, t_l, j - w0);
          if (in) {
            float ra[VW];
            load_run<VW>(qbase + static_cast<int64_t>(ta) * F + e, ra);
#pragma unroll
            for (int m = 0; m < VW; ++m) sum[m] = fmaf(ca, ra[m], sum[m]);
          }
        }
        if (in) store_run<VW>(grow + e, sum, !whole);
      }
      i = end;
    }
  }
}

// C[M][N] = sum_k A(m, k) B(k, n) on CUDA cores, fp32 accumulation; A is fp32 with
// element strides (sam, sak), B has the layer dtype with strides (sbk, sbn). 64 x 64
// tile per 256-thread block, 4 x 4 per thread, K staged 16 at a time; tiles load along
// whichever index is contiguous.
template <typename TB>
__global__ void __launch_bounds__(256) gemm_simt_kernel(
    const float* __restrict__ A, int64_t sam, int64_t sak, const TB* __restrict__ Bm, int64_t sbk,
    int64_t sbn, float* __restrict__ C, int64_t M, int64_t N, int64_t K) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 64, n0 = static_cast<int64_t>(blockIdx.x) * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      int mm, kk;
      if (sam == 1) { mm = i & 63; kk = i >> 6; } else { kk = i & 15; mm = i >> 4; }
      const int64_t gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * sam + gk * sak] : 0.f;
      int nn, kb;
      if (sbn == 1) { nn = i & 63; kb = i >> 6; } else { kb = i & 15; nn = i >> 4; }
      const int64_t gn = n0 + nn, gkb = k0 + kb;
      Bs[kb][nn] = (gn < N && gkb < K) ? load_elem(Bm, gkb * sbk + gn * sbn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t nn = n0 + tx * 4 + j;
      if (nn < N) C[m * N + nn] = acc[i][j];
    }
  }
}

// ------------------------------------------------------------------- launcher
static int64_t scan_blocks_of(int64_t slots) { return (slots + 4095) / 4096; }
static size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t backward_full_ws_bytes(const LayerArgs& a, bool tensor_path, FullBackwardWs* w, char* base) {
  const int64_t F = static_cast<int64_t>(a.H) * a.dq;
  const int64_t E = a.B * a.H * static_cast<int64_t>(a.k);
  const int64_t E2 = 2 * E > 0 ? 2 * E : 1;
  const int64_t tslots = 2LL * a.H * a.n;
  BackwardWs vws;
  size_t off = backward_ws_bytes(a.B, a.H, a.k, static_cast<int64_t>(a.n) * a.n, a.v, &vws,
                                base);
  const size_t o_gs = off;      off += al256(sizeof(float) * (E > 0 ? E : 1));
  const size_t o_acc = off;     off += al256(sizeof(float) * a.B * F);
  const size_t o_q = off;       off += al256(sizeof(float) * a.B * F);
  const size_t o_gq = off;      off += al256(sizeof(float) * a.B * F);
  const size_t o_gacc = off;    off += al256(tensor_path ? 0 : sizeof(float) * a.B * F);
  const size_t o_planes = off;  off += al256(tensor_path ? static_cast<size_t>(a.B) * F * 6 : 0);
  const size_t o_tg = off;      off += al256(sizeof(int) * E2);
  const size_t o_cf = off;      off += al256(sizeof(float) * E2);
  const size_t o_cnt = off;     off += al256(sizeof(int) * tslots);
  const size_t o_offs = off;    off += al256(sizeof(int) * (tslots + 1));
  const size_t o_part = off;    off += al256(sizeof(int) * (scan_blocks_of(tslots) + 1));
  const size_t o_ord = off;     off += al256(sizeof(int) * E2);
  const size_t o_bn = off;      off += al256(sizeof(float) * 2 * kBnChunks * F);
  const size_t o_sums = off;    off += al256(sizeof(float) * 2 * F);
  if (w && base) {
    w->values = vws;
    w->g_s = reinterpret_cast<float*>(base + o_gs);
    w->acc = reinterpret_cast<float*>(base + o_acc);
    w->q = reinterpret_cast<float*>(base + o_q);
    w->g_q = reinterpret_cast<float*>(base + o_gq);
    w->g_acc = tensor_path ? nullptr : reinterpret_cast<float*>(base + o_gacc);
    w->planes = tensor_path ? base + o_planes : nullptr;
    w->targets = reinterpret_cast<int*>(base + o_tg);
    w->coef = reinterpret_cast<float*>(base + o_cf);
    w->sub.counts = reinterpret_cast<int*>(base + o_cnt);
    w->sub.offsets = reinterpret_cast<int*>(base + o_offs);
    w->sub.partials = reinterpret_cast<int*>(base + o_part);
    w->sub.order = reinterpret_cast<int*>(base + o_ord);
    w->bn_part = reinterpret_cast<float*>(base + o_bn);
    w->bn_sums = reinterpret_cast<float*>(base + o_sums);
  }
  return off;
}

static unsigned grid_of(int64_t blocks, int64_t cap) {
  return static_cast<unsigned>(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

template <typename T, int VW>
static void launch_sub_kernels(const LayerArgs& a, const int* indices, uint16_t* g_planes,
                               const FullBackwardWs& w, cudaStream_t st) {
  const int64_t units = a.B * a.H;
  grad_q_targets_kernel<T, VW><<<grid_of((units + 3) / 4, 1LL << 30), 128, 0, st>>>(
      w.g_s, indices, static_cast<const T*>(a.subkeys), a.bn_gamma, a.bn_var, a.bn_eps, a.B, a.H,
      a.dq, a.n, a.k, w.g_q, w.g_acc, g_planes, w.targets, w.coef);
}

template <int VW>
static void launch_segment_subkeys(const LayerArgs& a, int64_t E2, int64_t tslots,
                                   float* grad_subkeys, const FullBackwardWs& w, cudaStream_t st) {
  const int64_t windows = (E2 + 31) / 32;
  segment_subkeys_kernel<VW><<<grid_of((windows + 3) / 4, 148 * 32), 128, 0, st>>>(
      w.sub.order, w.sub.offsets + tslots, w.targets, w.coef, w.q, a.H, a.dq, a.n, a.k,
      grad_subkeys);
}

template <typename T>
static cudaError_t launch_full_t(const LayerArgs& a, bool tensor_path, bool bn_training,
                                 const int* indices,
                                 const float* weights, const void* grad_out, float* grad_x,
                                 float* grad_W, float* grad_gamma, float* grad_beta,
                                 float* grad_subkeys, float* grad_scores,
                                 const FullBackwardWs& w, cudaStream_t st, int* launches) {
  const int64_t F = static_cast<int64_t>(a.H) * a.dq;
  const int64_t E = a.B * a.H * static_cast<int64_t>(a.k);
  const int64_t slots = static_cast<int64_t>(a.n) * a.n;
  const int half = a.dq / 2;
  const bool vec = (half % 8) == 0;
  cudaError_t e;
  // 1. kept-score gradients (into the workspace); the value gradients are launched by
  //    the caller.
  e = launch_grad_scores(a.B, a.H, a.k, a.v, a.dtype, slots, a.values, indices, weights,
                         grad_out, w.g_s, a.status, st);
  if (e != cudaSuccess) return e;
  *launches += 1;
  if (grad_scores) {
    e = cudaMemcpyAsync(grad_scores, w.g_s, sizeof(float) * E, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  // 2. acc = x W_q^T (the forward's query network without BatchNorm), q = BN(acc).
  LayerArgs raw = a;
  raw.raw_acc = 1;
  if (tensor_path) {
    e = launch_query_tc(raw, w.planes, st);
  } else {
    e = launch_query_bn_simt(raw, w.acc, st);
  }
  if (e != cudaSuccess) return e;
  const size_t aq_smem = F <= kAccQSmemF ? sizeof(float) * 2 * F : 0;
  acc_q_kernel<<<grid_of((a.B * F / 8 + 255) / 256, 148 * 8), 256, aq_smem, st>>>(
      tensor_path ? static_cast<const uint16_t*>(w.planes) : nullptr, w.acc, w.q, a.bn_mean,
      a.bn_var, a.bn_gamma, a.bn_beta, a.bn_eps, static_cast<int>(a.B), static_cast<int>(F));
  *launches += 2;
  // 3. dL/dq, dL/dacc (bf16 hi/lo planes for the tensor-core GEMMs), merged sub-key
  //    contributions.
  // The tensor-core layer shapes always suit the tensor-core GEMMs (the workspace holds
  // fp32 dL/dacc only for the CUDA-core path).
  const bool tc_gemm = tensor_path;
  if (tc_gemm && !gemm_tc_supported(a.B, static_cast<int>(F), a.d_model))
    return cudaErrorNotSupported;
  uint16_t* g_planes = tc_gemm ? static_cast<uint16_t*>(w.planes) : nullptr;
  // With batch statistics dL/dacc needs the column sums first; the kernel then
  // writes dL/dq only.
  FullBackwardWs wq = w;
  if (bn_training) wq.g_acc = nullptr;
  if (vec) launch_sub_kernels<T, 8>(a, indices, bn_training ? nullptr : g_planes, wq, st);
  else launch_sub_kernels<T, 1>(a, indices, bn_training ? nullptr : g_planes, wq, st);
  *launches += 1;
  // 4. BatchNorm: affine gradients (and, in training mode, dL/dacc).
  if (grad_gamma || grad_beta || bn_training) {
    dim3 g1(static_cast<unsigned>((F + 255) / 256), kBnChunks);
    bn_grad_partial_kernel<<<g1, 256, 0, st>>>(w.g_q, w.acc, a.bn_mean, a.bn_var, a.bn_eps, a.B,
                                               static_cast<int>(F), w.bn_part);
    bn_grad_final_kernel<<<static_cast<unsigned>((F + 31) / 32), kBnFinalWarps * 32, 0, st>>>(
        w.bn_part, static_cast<int>(F), grad_gamma, grad_beta, bn_training ? w.bn_sums : nullptr);
    *launches += 2;
  }
  if (bn_training) {
    e = launch_bn_train_dacc(w.g_q, w.acc, a.bn_mean, a.bn_var, a.bn_gamma, w.bn_sums, a.bn_eps,
                             a.B, static_cast<int>(F), tc_gemm ? nullptr : w.g_acc, g_planes, st);
    if (e != cudaSuccess) return e;
    *launches += 1;
  }
  // 5. Sub-key gradients: group the merged contributions by row, sum in windows.
  if (grad_subkeys) {
    const int64_t tslots = 2LL * a.H * a.n;
    const int64_t E2 = 2 * E;
    e = cudaMemsetAsync(grad_subkeys, 0, sizeof(float) * tslots * half, st);
    if (e != cudaSuccess) return e;
    // Merged-away picks carry target -1 and are skipped without a status.
    e = launch_counting_sort(w.targets, E2, tslots, w.sub, nullptr, st);
    if (e != cudaSuccess) return e;
    if (vec) launch_segment_subkeys<8>(a, E2, tslots, grad_subkeys, w, st);
    else launch_segment_subkeys<1>(a, E2, tslots, grad_subkeys, w, st);
    *launches += 6;
  }
  // 6. dL/dW_q = dL/dacc^T x  [F][d];  dL/dx = dL/dacc W_q  [B][d].
  if (tc_gemm) {
    if (grad_W) {
      e = launch_grad_w_tc(g_planes, a.x, grad_W, a.B, static_cast<int>(F), a.d_model, a.status,
                           st);
      if (e != cudaSuccess) return e;
      *launches += 1;
    }
    if (grad_x) {
      e = launch_grad_x_tc(g_planes, a.W_q, grad_x, a.B, static_cast<int>(F), a.d_model,
                           a.status, st);
      if (e != cudaSuccess) return e;
      *launches += 1;
    }
    return cudaGetLastError();
  }
  if (grad_W) {
    dim3 g(static_cast<unsigned>((a.d_model + 63) / 64), static_cast<unsigned>((F + 63) / 64));
    gemm_simt_kernel<T><<<g, 256, 0, st>>>(w.g_acc, 1, F, static_cast<const T*>(a.x), a.d_model,
                                           1, grad_W, F, a.d_model, a.B);
    *launches += 1;
  }
  if (grad_x) {
    dim3 g(static_cast<unsigned>((a.d_model + 63) / 64), static_cast<unsigned>((a.B + 63) / 64));
    gemm_simt_kernel<T><<<g, 256, 0, st>>>(w.g_acc, F, 1, static_cast<const T*>(a.W_q),
                                           a.d_model, 1, grad_x, a.B, a.d_model, F);
    *launches += 1;
  }
  return cudaGetLastError();
}

cudaError_t launch_backward_full(const LayerArgs& a, bool tensor_path, bool bn_training,
                                 const int* indices,
                                 const float* weights, const void* grad_out, float* grad_x,
                                 float* grad_W, float* grad_gamma, float* grad_beta,
                                 float* grad_subkeys, float* grad_values, float* grad_scores,
                                 const FullBackwardWs& w, const SideStream& side,
                                 cudaStream_t st, int* launches) {
  const int64_t slots = static_cast<int64_t>(a.n) * a.n;
  cudaError_t e = cudaSuccess;
  const bool split = grad_values && side.st;
  // The value gradients need only the picks and grad_out. The dependent chain of the
  // rest (kept-score gradients, query recompute, sub-key and BatchNorm sums, GEMMs) runs
  // on the helper stream, scheduled ahead of the caller's stream, and the value rows'
  // sort and row sums fill the SMs it leaves idle on the caller's stream.
  const cudaStream_t xs = split ? side.st : st;
  if (split) e = side_fork(side, st);
  if (e == cudaSuccess) {
    if (a.dtype == 0)
      e = launch_full_t<float>(a, tensor_path, bn_training, indices, weights, grad_out, grad_x,
                               grad_W, grad_gamma, grad_beta, grad_subkeys, grad_scores, w, xs,
                               launches);
    else
      e = launch_full_t<uint16_t>(a, tensor_path, bn_training, indices, weights, grad_out,
                                  grad_x, grad_W, grad_gamma, grad_beta, grad_subkeys,
                                  grad_scores, w, xs, launches);
  }
  if (grad_values) {
    if (e == cudaSuccess)
      e = launch_value_rows(a.B, a.H, a.k, a.v, a.dtype, slots, indices, weights, grad_out,
                            grad_values, w.values, a.status, st);
    *launches += backward_values_launches(slots, false, true);
  }
  // Always join, even after an error, so the caller's stream never runs ahead of work
  // already queued on the side stream.
  if (split) {
    const cudaError_t e2 = side_join(side, st);
    if (e == cudaSuccess) e = e2;
  }
  return e;
}

}  // namespace pkm
