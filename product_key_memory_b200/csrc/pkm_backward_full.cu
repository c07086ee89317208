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
#include "pkm_common.cuh"
#include "pkm_kernels.h"
#include "pkm_tc.h"

namespace pkm {

// acc = hi + mid + lo from the three bf16 planes the tensor-core query kernel writes.
__global__ void planes_to_acc_kernel(const uint16_t* __restrict__ planes, int64_t count,
                                     float* __restrict__ acc) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float hi = load_elem(planes, i), mid = load_elem(planes, count + i);
    const float lo = load_elem(planes, 2 * count + i);
    acc[i] = hi + mid + lo;
  }
}

// dL/dq and dL/dacc for one token per warp. g_s [B][H][k] are the kept-score gradients.
template <typename T>
__global__ void __launch_bounds__(128) grad_q_kernel(
    const float* __restrict__ g_s, const int* __restrict__ indices, const T* __restrict__ subkeys,
    const float* __restrict__ gamma, const float* __restrict__ var, float eps, int64_t B, int H,
    int dq, int n, int k, float* __restrict__ g_q, float* __restrict__ g_acc) {
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= B) return;
  const int half = dq / 2, F = H * dq;
  const int64_t slots = static_cast<int64_t>(n) * n;
  for (int h = 0; h < H; ++h) {
    const int64_t base = (t * H + h) * static_cast<int64_t>(k);
    for (int side = 0; side < 2; ++side) {
      const int f0 = h * dq + side * half;
      for (int e0 = 0; e0 < half; e0 += 32 * 8) {
        float acc[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m] = 0.f;
        for (int j = 0; j < k; ++j) {
          const int slot = indices[base + j];
          if (slot < 0 || slot >= slots) continue;
          const int sub = side ? slot % n : slot / n;
          const float g = g_s[base + j];
          const T* row = subkeys + (static_cast<int64_t>(h * 2 + side) * n + sub) * half;
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int e = e0 + lane + 32 * m;
            if (e < half) acc[m] = fmaf(g, load_elem(row, e), acc[m]);
          }
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int e = e0 + lane + 32 * m;
          if (e < half) {
            const int f = f0 + e;
            g_q[t * F + f] = acc[m];
            g_acc[t * F + f] = acc[m] * (gamma[f] / sqrtf(var[f] + eps));
          }
        }
      }
    }
  }
}

// Column sums over tokens, pass 1: block (feature group of 256, token chunk) writes its
// partial dL/dbeta and dL/dgamma sums; pass 2 adds the chunks in a fixed order.
constexpr int kBnChunks = 32;

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
  for (int64_t t = t0; t < t1; ++t) {
    const float g = g_q[t * F + f];
    sb += g;
    sg = fmaf(g, (acc[t * F + f] - mu) * rs, sg);
  }
  part[static_cast<int64_t>(blockIdx.y) * 2 * F + f] = sb;
  part[static_cast<int64_t>(blockIdx.y) * 2 * F + F + f] = sg;
}

__global__ void bn_grad_final_kernel(const float* __restrict__ part, int F,
                                     float* __restrict__ grad_gamma, float* __restrict__ grad_beta) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= F) return;
  float sb = 0.f, sg = 0.f;
  for (int c = 0; c < kBnChunks; ++c) {
    sb += part[static_cast<int64_t>(c) * 2 * F + f];
    sg += part[static_cast<int64_t>(c) * 2 * F + F + f];
  }
  if (grad_beta) grad_beta[f] = sb;
  if (grad_gamma) grad_gamma[f] = sg;
}

// Each pick feeds two sub-keys: target 2e = left (h, 0, i), 2e + 1 = right (h, 1, i').
__global__ void subkey_targets_kernel(const int* __restrict__ indices, int64_t E, int H, int n,
                                      int k, int* __restrict__ targets) {
  const int64_t slots = static_cast<int64_t>(n) * n;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < E;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int slot = indices[e];
    const int h = static_cast<int>((e / k) % H);
    const bool ok = slot >= 0 && slot < slots;
    targets[2 * e] = ok ? (h * 2) * n + slot / n : -1;
    targets[2 * e + 1] = ok ? (h * 2 + 1) * n + slot % n : -1;
  }
}

// Windows of 32 sorted contributions per warp; a contribution adds g_c * q_half[t] to
// its sub-key's gradient row. Groups inside a window are written once (the table was
// zeroed); groups crossing a window edge use atomics.
__global__ void __launch_bounds__(128) segment_subkeys_kernel(
    const int* __restrict__ order, const int* __restrict__ offsets,
    const int* __restrict__ total_ptr, const int* __restrict__ targets,
    const float* __restrict__ g_s, const float* __restrict__ acc, const float* __restrict__ mean,
    const float* __restrict__ var, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, int H, int dq, int n, int k,
    float* __restrict__ grad_subkeys) {
  const int lane = threadIdx.x & 31;
  const int total = *total_ptr;
  const int half = dq / 2, F = H * dq, HK = H * k;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t win = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       win * 32 < total; win += nwarps) {
    const int w0 = static_cast<int>(win * 32);
    const int w1 = min(w0 + 32, total);
    int c_l = 0, tg_l = 0;
    if (w0 + lane < w1) {
      c_l = order[w0 + lane];
      tg_l = targets[c_l];
    }
    int i = w0;
    while (i < w1) {
      const int tg = __shfl_sync(0xffffffffu, tg_l, i - w0);
      const int seg0 = offsets[tg], seg1 = offsets[tg + 1];
      const int end = min(seg1, w1);
      const bool whole = seg0 >= w0 && seg1 <= w1;
      const int side = (tg / n) & 1;
      const int h = tg / (2 * n);
      float* grow = grad_subkeys + static_cast<int64_t>(tg) * half;
      for (int e0 = 0; e0 < half; e0 += 32 * 8) {
        float sum[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) sum[m] = 0.f;
        for (int j = i; j < end; ++j) {
          const int c = __shfl_sync(0xffffffffu, c_l, j - w0);
          const int e = c >> 1;
          const int64_t t = e / HK;
          const float g = g_s[e];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int ee = e0 + lane + 32 * m;
            if (ee < half) {
              const int f = h * dq + side * half + ee;
              const float q = (acc[t * F + f] - mean[f]) * (gamma[f] / sqrtf(var[f] + eps)) + beta[f];
              sum[m] = fmaf(g, q, sum[m]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int ee = e0 + lane + 32 * m;
          if (ee < half) {
            if (whole) grow[ee] += sum[m];
            else atomicAdd(grow + ee, sum[m]);
          }
        }
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
  const int64_t tslots = 2LL * a.H * a.n;
  BackwardWs vws;
  size_t off = backward_ws_bytes(a.B, a.H, a.k, static_cast<int64_t>(a.n) * a.n, &vws, base);
  const size_t o_gs = off;      off += al256(sizeof(float) * (E > 0 ? E : 1));
  const size_t o_acc = off;     off += al256(sizeof(float) * a.B * F);
  const size_t o_gq = off;      off += al256(sizeof(float) * a.B * F);
  const size_t o_gacc = off;    off += al256(sizeof(float) * a.B * F);
  const size_t o_planes = off;  off += al256(tensor_path ? static_cast<size_t>(a.B) * F * 6 : 0);
  const size_t o_tg = off;      off += al256(sizeof(int) * (2 * E > 0 ? 2 * E : 1));
  const size_t o_cnt = off;     off += al256(sizeof(int) * tslots);
  const size_t o_offs = off;    off += al256(sizeof(int) * (tslots + 1));
  const size_t o_part = off;    off += al256(sizeof(int) * (scan_blocks_of(tslots) + 1));
  const size_t o_ord = off;     off += al256(sizeof(int) * (2 * E > 0 ? 2 * E : 1));
  const size_t o_bn = off;      off += al256(sizeof(float) * 2 * kBnChunks * F);
  if (w && base) {
    w->values = vws;
    w->g_s = reinterpret_cast<float*>(base + o_gs);
    w->acc = reinterpret_cast<float*>(base + o_acc);
    w->g_q = reinterpret_cast<float*>(base + o_gq);
    w->g_acc = reinterpret_cast<float*>(base + o_gacc);
    w->planes = base + o_planes;
    w->targets = reinterpret_cast<int*>(base + o_tg);
    w->sub.counts = reinterpret_cast<int*>(base + o_cnt);
    w->sub.offsets = reinterpret_cast<int*>(base + o_offs);
    w->sub.partials = reinterpret_cast<int*>(base + o_part);
    w->sub.order = reinterpret_cast<int*>(base + o_ord);
    w->bn_part = reinterpret_cast<float*>(base + o_bn);
  }
  return off;
}

template <typename T>
static cudaError_t launch_full_t(const LayerArgs& a, bool tensor_path, const int* indices,
                                 const float* weights, const void* grad_out, float* grad_x,
                                 float* grad_W, float* grad_gamma, float* grad_beta,
                                 float* grad_subkeys, float* grad_values, float* grad_scores,
                                 const FullBackwardWs& w, cudaStream_t st, int* launches) {
  const int64_t F = static_cast<int64_t>(a.H) * a.dq;
  const int64_t E = a.B * a.H * static_cast<int64_t>(a.k);
  const int64_t slots = static_cast<int64_t>(a.n) * a.n;
  cudaError_t e;
  // 1. kept-score gradients (into the workspace) and, if asked, the value gradients.
  e = launch_backward_values(a.B, a.H, a.k, a.v, a.dtype, slots, a.values, indices, weights,
                             grad_out, grad_values, w.g_s, w.values, a.status, st, [] {});
  if (e != cudaSuccess) return e;
  *launches += grad_values ? 7 : 1;
  if (grad_scores) {
    e = cudaMemcpyAsync(grad_scores, w.g_s, sizeof(float) * E, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  // 2. acc = x W_q^T (the forward's query network without BatchNorm).
  LayerArgs raw = a;
  raw.raw_acc = 1;
  if (tensor_path) {
    e = launch_query_tc(raw, w.planes, st);
    if (e != cudaSuccess) return e;
    const int64_t cnt = a.B * F;
    const int64_t blocks = (cnt + 255) / 256;
    planes_to_acc_kernel<<<static_cast<unsigned>(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, st>>>(
        static_cast<const uint16_t*>(w.planes), cnt, w.acc);
    *launches += 2;
  } else {
    e = launch_query_bn_simt(raw, w.acc, st);
    if (e != cudaSuccess) return e;
    *launches += 1;
  }
  // 3. dL/dq, dL/dacc.
  grad_q_kernel<T><<<static_cast<unsigned>((a.B + 3) / 4), 128, 0, st>>>(
      w.g_s, indices, static_cast<const T*>(a.subkeys), a.bn_gamma, a.bn_var, a.bn_eps, a.B, a.H,
      a.dq, a.n, a.k, w.g_q, w.g_acc);
  *launches += 1;
  // 4. BatchNorm affine gradients.
  if (grad_gamma || grad_beta) {
    dim3 g1(static_cast<unsigned>((F + 255) / 256), kBnChunks);
    bn_grad_partial_kernel<<<g1, 256, 0, st>>>(w.g_q, w.acc, a.bn_mean, a.bn_var, a.bn_eps, a.B,
                                               static_cast<int>(F), w.bn_part);
    bn_grad_final_kernel<<<static_cast<unsigned>((F + 255) / 256), 256, 0, st>>>(
        w.bn_part, static_cast<int>(F), grad_gamma, grad_beta);
    *launches += 2;
  }
  // 5. Sub-key gradients: group the 2E contributions by sub-key, sum in windows.
  if (grad_subkeys) {
    const int64_t tslots = 2LL * a.H * a.n;
    const int64_t E2 = 2 * E;
    e = cudaMemsetAsync(grad_subkeys, 0, sizeof(float) * tslots * (a.dq / 2), st);
    if (e != cudaSuccess) return e;
    const int64_t eb = (E + 255) / 256;
    subkey_targets_kernel<<<static_cast<unsigned>(eb < 148 * 16 ? eb : 148 * 16), 256, 0, st>>>(
        indices, E, a.H, a.n, a.k, w.targets);
    e = launch_counting_sort(w.targets, E2, tslots, w.sub, a.status, st);
    if (e != cudaSuccess) return e;
    const int64_t windows = (E2 + 31) / 32;
    const int64_t sblocks = (windows + 3) / 4;
    segment_subkeys_kernel<<<static_cast<unsigned>(sblocks < 148 * 32 ? (sblocks > 0 ? sblocks : 1) : 148 * 32), 128, 0, st>>>(
        w.sub.order, w.sub.offsets, w.sub.offsets + tslots, w.targets, w.g_s, w.acc, a.bn_mean,
        a.bn_var, a.bn_gamma, a.bn_beta, a.bn_eps, a.H, a.dq, a.n, a.k, grad_subkeys);
    *launches += 7;
  }
  // 6. dL/dW_q = dL/dacc^T x  [F][d];  dL/dx = dL/dacc W_q  [B][d].
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

cudaError_t launch_backward_full(const LayerArgs& a, bool tensor_path, const int* indices,
                                 const float* weights, const void* grad_out, float* grad_x,
                                 float* grad_W, float* grad_gamma, float* grad_beta,
                                 float* grad_subkeys, float* grad_values, float* grad_scores,
                                 const FullBackwardWs& w, cudaStream_t st, int* launches) {
  if (a.dtype == 0)
    return launch_full_t<float>(a, tensor_path, indices, weights, grad_out, grad_x, grad_W,
                                grad_gamma, grad_beta, grad_subkeys, grad_values, grad_scores, w,
                                st, launches);
  return launch_full_t<uint16_t>(a, tensor_path, indices, weights, grad_out, grad_x, grad_W,
                                 grad_gamma, grad_beta, grad_subkeys, grad_values, grad_scores, w,
                                 st, launches);
}

}  // namespace pkm
