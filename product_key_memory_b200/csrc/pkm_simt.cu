// pkm_simt.cu -- CUDA-core (SIMT, fp32) kernels for the query network and the
// per-half sub-key search. They serve fp32 layers and any shape the tensor-core
// kernels do not take.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology and the
// Deep Analysis / Methodology list): the query network q(x) is a linear map with
// BatchNorm; q is split into halves q1, q2; each half is scored against its own
// sub-key set and the top-k sub-keys of each half are kept.
#include "pkm_common.cuh"
#include "pkm_kernels.h"

namespace pkm {

// ---------------------------------------------------------------------------
// q[t][f] = (sum_c x[t][c] W[f][c] - mean[f]) * gamma[f] / sqrt(var[f] + eps) + beta[f]
// 64 x 64 output tile per 256-thread block, 4 x 4 per thread, K staged 16 at a time.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) query_bn_simt_kernel(
    const T* __restrict__ x, const T* __restrict__ W, const float* __restrict__ mean,
    const float* __restrict__ var, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, int64_t B, int d, int F,
    float* __restrict__ q, int raw_acc) {
  __shared__ float xs[16][64 + 4];
  __shared__ float ws[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 64;
  const int n0 = blockIdx.x * 64;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < d; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i >> 4, c = i & 15;
      const int64_t gm = m0 + r;
      const int gk = k0 + c;
      xs[c][r] = (gm < B && gk < d) ? load_elem(x, gm * d + gk) : 0.f;
      const int gn = n0 + r;
      ws[c][r] = (gn < F && gk < d) ? load_elem(W, static_cast<int64_t>(gn) * d + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int f = n0 + tx * 4 + j;
    if (f >= F) continue;
    const float scale = raw_acc ? 1.f : gamma[f] / sqrtf(var[f] + eps);
    const float mu = raw_acc ? 0.f : mean[f], bt = raw_acc ? 0.f : beta[f];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t m = m0 + ty * 4 + i;
      if (m < B) q[m * F + f] = (acc[i][j] - mu) * scale + bt;
    }
  }
}

// ---------------------------------------------------------------------------
// Per-half sub-key scores and top-k. Block = (32 tokens, one head, one half):
// 8 warps x 4 tokens. Sub-keys are staged 32 rows at a time in shared memory;
// lane i scores sub-key (chunk + i) for each of the warp's tokens, and the warp
// keeps a sorted best-32 list per token (one entry per lane) with sort + merge.
// Output: list_s / list_i [B][H][2][32]: the best 32 of each half (best first here;
// padding entries have score -inf and id kIdPad when n < 32).
// ---------------------------------------------------------------------------
constexpr int kSimtTokPerWarp = 4;
constexpr int kSimtWarps = 8;
constexpr int kSimtTok = kSimtTokPerWarp * kSimtWarps;

template <typename T>
__global__ void __launch_bounds__(kSimtWarps * 32) subkey_topk_simt_kernel(
    const float* __restrict__ q, const T* __restrict__ subkeys, int64_t B, int H, int dq,
    int n, int k, float* __restrict__ list_s, int* __restrict__ list_i) {
  extern __shared__ float smem[];
  const int half = dq >> 1;
  const int ld = half + 1;                       // padded row: conflict-free column reads
  float* keys = smem;                            // [32][ld]
  float* qs = smem + 32 * ld;                    // [kSimtTok][half]
  const int hs = blockIdx.y;                     // h * 2 + side
  const int h = hs >> 1, side = hs & 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kSimtTok;
  const int F = 2 * half * H;

  for (int i = threadIdx.x; i < kSimtTok * half; i += blockDim.x) {
    const int r = i / half, e = i - r * half;
    const int64_t t = t0 + r;
    qs[i] = (t < B) ? q[t * F + h * dq + side * half + e] : 0.f;
  }
  float best_s[kSimtTokPerWarp];
  int best_i[kSimtTokPerWarp];
#pragma unroll
  for (int u = 0; u < kSimtTokPerWarp; ++u) { best_s[u] = -INFINITY; best_i[u] = kIdPad; }

  const T* book = subkeys + static_cast<int64_t>(hs) * n * half;
  for (int c0 = 0; c0 < n; c0 += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * half; i += blockDim.x) {
      const int r = i / half, e = i - r * half;
      keys[r * ld + e] = (c0 + r < n) ? load_elem(book, static_cast<int64_t>(c0 + r) * half + e) : 0.f;
    }
    __syncthreads();
    const bool valid = c0 + lane < n;
#pragma unroll
    for (int u = 0; u < kSimtTokPerWarp; ++u) {
      const float* qq = qs + (warp * kSimtTokPerWarp + u) * half;
      const float* kk = keys + lane * ld;
      float acc = 0.f;
      for (int e = 0; e < half; ++e) acc = fmaf(qq[e], kk[e], acc);
      float cs = valid ? acc : -INFINITY;
      int ci = valid ? c0 + lane : kIdPad;
      // Skip the merge when no new score beats the current 32nd best.
      const float ks = __shfl_sync(0xffffffffu, best_s[u], 31);
      const int ki = __shfl_sync(0xffffffffu, best_i[u], 31);
      if (__any_sync(0xffffffffu, better(cs, ci, ks, ki))) {
        warp_sort32(cs, ci);
        warp_merge32(best_s[u], best_i[u], cs, ci);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kSimtTokPerWarp; ++u) {
    const int64_t t = t0 + warp * kSimtTokPerWarp + u;
    if (t < B) {
      const int64_t o = ((t * H + h) * 2 + side) * kMaxK + lane;
      list_s[o] = best_s[u];
      list_i[o] = best_i[u];
    }
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_query_bn_simt(const LayerArgs& a, float* q, cudaStream_t st) {
  const int F = a.H * a.dq;
  dim3 grid((F + 63) / 64, static_cast<unsigned>((a.B + 63) / 64));
  if (a.dtype == 0)
    query_bn_simt_kernel<float><<<grid, 256, 0, st>>>(
        static_cast<const float*>(a.x), static_cast<const float*>(a.W_q), a.bn_mean, a.bn_var,
        a.bn_gamma, a.bn_beta, a.bn_eps, a.B, a.d_model, F, q, a.raw_acc);
  else
    query_bn_simt_kernel<uint16_t><<<grid, 256, 0, st>>>(
        static_cast<const uint16_t*>(a.x), static_cast<const uint16_t*>(a.W_q), a.bn_mean,
        a.bn_var, a.bn_gamma, a.bn_beta, a.bn_eps, a.B, a.d_model, F, q, a.raw_acc);
  return cudaGetLastError();
}

size_t subkey_topk_simt_smem(int dq) {
  const int half = dq / 2;
  return sizeof(float) * (32 * (half + 1) + kSimtTok * half);
}

cudaError_t launch_subkey_topk_simt(const LayerArgs& a, const float* q, float* list_s,
                                    int* list_i, cudaStream_t st) {
  const size_t smem = subkey_topk_simt_smem(a.dq);
  dim3 grid(static_cast<unsigned>((a.B + kSimtTok - 1) / kSimtTok), a.H * 2);
  cudaError_t e;
  if (a.dtype == 0) {
    e = set_max_smem(reinterpret_cast<const void*>(subkey_topk_simt_kernel<float>), smem);
    if (e != cudaSuccess) return e;
    subkey_topk_simt_kernel<float><<<grid, kSimtWarps * 32, smem, st>>>(
        q, static_cast<const float*>(a.subkeys), a.B, a.H, a.dq, a.n, a.k, list_s, list_i);
  } else {
    e = set_max_smem(reinterpret_cast<const void*>(subkey_topk_simt_kernel<uint16_t>), smem);
    if (e != cudaSuccess) return e;
    subkey_topk_simt_kernel<uint16_t><<<grid, kSimtWarps * 32, smem, st>>>(
        q, static_cast<const uint16_t*>(a.subkeys), a.B, a.H, a.dq, a.n, a.k, list_s, list_i);
  }
  return cudaGetLastError();
}

}  // namespace pkm
