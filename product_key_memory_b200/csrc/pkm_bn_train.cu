// pkm_bn_train.cu -- BatchNorm of the query network in training mode.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology: the
// query network has batch normalization). While the model trains, the batch's own
// statistics normalise it (Ioffe and Szegedy 2015):
//   mean_B = (1/B) sum_t acc[t],  var_B = (1/B) sum_t (acc[t] - mean_B)^2
// and the running statistics move towards them with momentum m:
//   running_mean <- (1 - m) running_mean + m mean_B
//   running_var  <- (1 - m) running_var  + m var_B B / (B - 1)
// In the backward the statistics depend on every token:
//   dL/dacc = gamma / sqrt(var_B + eps) (g - (1/B) sum_t g - xhat (1/B) sum_t g xhat),
//   g = dL/dq, xhat = (acc - mean_B) / sqrt(var_B + eps).
#include <cuda_bf16.h>

#include "pkm_common.cuh"
#include "pkm_kernels.h"

namespace pkm {

// Pass 1: per (256 features, chunk of kStatChunk tokens), fp64 chunk mean and sum of
// squared deviations from it (two passes over the chunk; the second one hits cache).
// acc comes as three bf16 planes (hi + mid + lo) or as fp32.
__global__ void __launch_bounds__(256) bn_stats_partial_kernel(
    const uint16_t* __restrict__ planes, const float* __restrict__ acc, int B, int F,
    double* __restrict__ part) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= F) return;
  const int t0 = blockIdx.y * kStatChunk, t1 = min(B, t0 + kStatChunk);
  const int64_t count = static_cast<int64_t>(B) * F;
  auto value = [&](int t) -> double {
    const int64_t i = static_cast<int64_t>(t) * F + f;
    if (planes)
      return static_cast<double>(load_elem(planes, i) + load_elem(planes, count + i) +
                                 load_elem(planes, 2 * count + i));
    return static_cast<double>(acc[i]);
  };
  double s = 0.0;
  for (int t = t0; t < t1; ++t) s += value(t);
  const double mu = s / (t1 - t0);
  double m2 = 0.0;
  for (int t = t0; t < t1; ++t) {
    const double dv = value(t) - mu;
    m2 = fma(dv, dv, m2);
  }
  part[(static_cast<int64_t>(blockIdx.y) * 2) * F + f] = mu;
  part[(static_cast<int64_t>(blockIdx.y) * 2 + 1) * F + f] = m2;
}

// Chan, Golub and LeVeque's pairwise update: (n, mean, m2) absorbs (nb, mb, m2b).
__device__ __forceinline__ void chan_merge(double& n, double& mean, double& m2, double nb,
                                           double mb, double m2b) {
  if (nb == 0.0) return;
  const double tot = n + nb;
  const double delta = mb - mean;
  mean += delta * (nb / tot);
  m2 += m2b + delta * delta * (n * nb / tot);
  n = tot;
}

// Pass 2: block = 32 features x 8 warps; warp w merges its share of the chunks in
// order, then warp 0 merges the 8 warp results in order (a fixed order:
// deterministic). Writes the batch statistics and moves the running ones.
constexpr int kStatWarps = 8;

__global__ void __launch_bounds__(kStatWarps * 32) bn_stats_final_kernel(
    const double* __restrict__ part, int B, int F, float momentum,
    float* __restrict__ batch_mean, float* __restrict__ batch_var,
    float* __restrict__ running_mean, float* __restrict__ running_var) {
  __shared__ double sn[kStatWarps][32], sm[kStatWarps][32], s2[kStatWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * 32 + lane;
  const int chunks = (B + kStatChunk - 1) / kStatChunk;
  const int per = (chunks + kStatWarps - 1) / kStatWarps;
  double n = 0.0, mean = 0.0, m2 = 0.0;
  if (f < F) {
    for (int c = warp * per; c < min(chunks, (warp + 1) * per); ++c) {
      const double nb = static_cast<double>(min(B, (c + 1) * kStatChunk) - c * kStatChunk);
      chan_merge(n, mean, m2, nb, part[(static_cast<int64_t>(c) * 2) * F + f],
                 part[(static_cast<int64_t>(c) * 2 + 1) * F + f]);
    }
  }
  sn[warp][lane] = n;
  sm[warp][lane] = mean;
  s2[warp][lane] = m2;
  __syncthreads();
  if (warp != 0 || f >= F) return;
  n = 0.0;
  mean = 0.0;
  m2 = 0.0;
  for (int w = 0; w < kStatWarps; ++w) chan_merge(n, mean, m2, sn[w][lane], sm[w][lane], s2[w][lane]);
  const double var = m2 / B;
  batch_mean[f] = static_cast<float>(mean);
  batch_var[f] = static_cast<float>(var);
  const double m = momentum;
  running_mean[f] = static_cast<float>((1.0 - m) * running_mean[f] + m * mean);
  running_var[f] = static_cast<float>((1.0 - m) * running_var[f] + m * (m2 / (B - 1)));
}

cudaError_t launch_bn_batch_stats(const uint16_t* planes, const float* acc, int64_t B, int F,
                                  float momentum, double* part, float* batch_mean,
                                  float* batch_var, float* running_mean, float* running_var,
                                  cudaStream_t st) {
  const int chunks = static_cast<int>((B + kStatChunk - 1) / kStatChunk);
  dim3 g1((F + 255) / 256, chunks);
  bn_stats_partial_kernel<<<g1, 256, 0, st>>>(planes, acc, static_cast<int>(B), F, part);
  bn_stats_final_kernel<<<(F + 31) / 32, kStatWarps * 32, 0, st>>>(
      part, static_cast<int>(B), F, momentum, batch_mean, batch_var, running_mean, running_var);
  return cudaGetLastError();
}

// dL/dacc with batch statistics, from g = dL/dq, acc and the column sums
// sums[0][f] = sum_t g, sums[1][f] = sum_t g xhat. Written as fp32 (g_acc) and/or bf16
// hi/lo planes [2][B][F] for the tensor-core GEMMs. Thread = one feature (its BN
// constants in registers), rows strided over grid.y.
__global__ void __launch_bounds__(256) bn_train_dacc_kernel(
    const float* __restrict__ g_q, const float* __restrict__ acc,
    const float* __restrict__ mean, const float* __restrict__ var,
    const float* __restrict__ gamma, const float* __restrict__ sums, float eps, int B, int F,
    float* __restrict__ g_acc, uint16_t* __restrict__ g_planes) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= F) return;
  const int64_t count = static_cast<int64_t>(B) * F;
  const float inv_b = 1.f / static_cast<float>(B);
  const float rs = 1.f / sqrtf(var[f] + eps);
  const float mu = mean[f], gs = gamma[f] * rs;
  const float mb = sums[f] * inv_b, mg = sums[F + f] * inv_b;
  for (int t = blockIdx.y; t < B; t += gridDim.y) {
    const int64_t i = static_cast<int64_t>(t) * F + f;
    const float xhat = (acc[i] - mu) * rs;
    const float ga = gs * (g_q[i] - mb - xhat * mg);
    if (g_acc) g_acc[i] = ga;
    if (g_planes) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(ga);
      const __nv_bfloat16 lo = __float2bfloat16_rn(ga - __bfloat162float(hi));
      g_planes[i] = __bfloat16_as_ushort(hi);
      g_planes[count + i] = __bfloat16_as_ushort(lo);
    }
  }
}

cudaError_t launch_bn_train_dacc(const float* g_q, const float* acc, const float* mean,
                                 const float* var, const float* gamma, const float* sums,
                                 float eps, int64_t B, int F, float* g_acc, uint16_t* g_planes,
                                 cudaStream_t st) {
  const unsigned gx = static_cast<unsigned>((F + 255) / 256);
  const unsigned gy = static_cast<unsigned>(B < 1024 ? B : 1024);
  bn_train_dacc_kernel<<<dim3(gx, gy), 256, 0, st>>>(g_q, acc, mean, var, gamma, sums, eps,
                                                     static_cast<int>(B), F, g_acc, g_planes);
  return cudaGetLastError();
}

}  // namespace pkm
