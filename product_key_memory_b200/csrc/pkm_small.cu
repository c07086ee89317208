// pkm_small.cu -- the forward for small batches (B <= kSmallMaxB tokens): the
// serving case of one or a few sequences' tokens, where latency rather than HBM
// bandwidth is the goal ("Large Memory Layers with Product Keys", gptget.net
// summary: the memory layer makes inference faster than a larger dense model).
//
// The large-batch kernels tile 128 tokens per CTA, so a handful of tokens leaves
// almost every SM idle and each stage is bound by one SM's bandwidth. Here every
// stage spreads the layer's parameters over the whole GPU instead, in three kernels
// chained by programmatic dependent launch:
//   query   q = BN(x W_q^T). Decode mode (a few tokens): query_decode_kernel, a warp
//           per W_q row for all tokens. bf16 layers above it: query_mma_kernel, CTA =
//           16 features x 16 tokens as warp-level tensor-core tiles. Otherwise (fp32):
//           query_small_kernel, CTA = 16 features x 8 tokens, one warp per token.
//   scores  the per-half scores of 64-sub-key chunks and each token's best 32 of a
//           chunk: score_decode_kernel (a warp per 8 sub-keys, all tokens),
//           score_mma_kernel (CTA = 64 sub-keys x 16 tokens, tensor-core tiles),
//           score_small_kernel (CTA = 64 sub-keys x 16 tokens, a lane per sub-key)
//   gather  gather_small_kernel, CTA = (token, head), the H heads of a token one
//           cluster: merge the chunk lists of each half, exact top-k of the pruned
//           candidates, softmax, the head's k weighted value rows over 8 warps, heads
//           summed over distributed shared memory
// forward_small_fused_kernel runs the same three stages as one cooperative launch.
// fp32 q and fp32 dot products (fp32 accumulation of bf16 products on the tensor
// cores, q split into two bf16 planes for the scores); the selection order and the
// candidate pruning of the large-batch path.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "pkm_common.cuh"
#include "pkm_kernels.h"
#include "pkm_select.cuh"
#include "pkm_tc.h"
#include "pkm_tcgen05.cuh"

namespace pkm {

constexpr int kQFeat = 16;        // features per query CTA
constexpr int kSChunk = 64;       // sub-keys per scoring CTA
constexpr int kSTok = 16;         // tokens per scoring CTA (2 per warp)
constexpr int kSmallWarps = 8;
constexpr int kQTok = kSmallWarps;  // tokens per query CTA (one per warp)

// Programmatic dependent launch: the next kernel on the stream may start launching
// once every CTA of this one has passed launch_dependents; its CTAs block in
// wait_prior_grid until this grid has finished and its writes are visible.
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Prologue of the three-kernel form's first kernel, which is itself launched as a
// programmatic dependent: its CTAs can be resident before the stream's previous kernel
// ends, and wait here until that kernel's writes are visible (x and the parameters may
// come from it). Then it clears the call's status word (clear, when the caller asks for
// it instead of a memset before the launch) and lets the scoring kernel launch.
__device__ __forceinline__ void first_kernel_prologue(int* clear) {
  wait_prior_grid();
  if (clear && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *clear = 0;
  allow_dependents();
}

// Copy `words` 32-bit words from global to shared memory with every thread keeping
// kCopyDepth loads in flight (the staging loops otherwise serialise on latency).
// Row r of `rows` words lands at dst + r * dst_ld; rows at or past `valid_rows` are
// zero-filled.
constexpr int kCopyDepth = 8;

__device__ __forceinline__ void stage_rows(const uint32_t* __restrict__ src, uint32_t* dst,
                                           int nrows, int valid_rows, int row_words,
                                           int dst_ld) {
  if ((row_words & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    // 16-byte loads (four words of one row each), stored as words (rows may be padded).
    const int row_vecs = row_words >> 2;
    const int total = nrows * row_vecs;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    for (int base = threadIdx.x; base < total; base += blockDim.x * kCopyDepth) {
      uint4 v[kCopyDepth];
#pragma unroll
      for (int u = 0; u < kCopyDepth; ++u) {
        const int i = base + u * blockDim.x;
        const int r = i / row_vecs;
        v[u] = (i < total && r < valid_rows) ? __ldg(s4 + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kCopyDepth; ++u) {
        const int i = base + u * blockDim.x;
        if (i < total) {
          const int r = i / row_vecs;
          uint32_t* d = dst + r * dst_ld + ((i - r * row_vecs) << 2);
          d[0] = v[u].x; d[1] = v[u].y; d[2] = v[u].z; d[3] = v[u].w;
        }
      }
    }
    return;
  }
  const int total = nrows * row_words;
  for (int base = threadIdx.x; base < total; base += blockDim.x * kCopyDepth) {
    uint32_t v[kCopyDepth];
#pragma unroll
    for (int u = 0; u < kCopyDepth; ++u) {
      const int i = base + u * blockDim.x;
      const int r = i / row_words;
      v[u] = (i < total && r < valid_rows) ? __ldg(src + i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kCopyDepth; ++u) {
      const int i = base + u * blockDim.x;
      if (i < total) {
        const int r = i / row_words;
        dst[r * dst_ld + (i - r * row_words)] = v[u];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Decode mode: batches of at most kDecodeB tokens. The kernels below give each warp a
// token, so with one token a single warp of every block does that block's work. In
// decode mode a warp instead takes one W_q row (query) or kDecodeKeys sub-keys
// (scoring) for every token, its lanes splitting the contraction: lane L reads the
// 16-byte chunks L, L + 32, ... of each row straight from global memory, all in flight
// together, and accumulates their elements in order with fmaf; the lanes' partial sums
// are then added by an xor tree over lane masks 16, 8, 4, 2, 1 (every lane ends with
// the same total). Both small-batch forms use these functions and the same decode_mode
// test, so their results stay identical.
// ---------------------------------------------------------------------------
constexpr int kDecodeB = 8;        // decode mode's largest batch
constexpr int kDecodeRowVecs = 8;  // 16-byte chunks per lane of a W_q row: d*esz <= 4 KiB
constexpr int kDecodeKeyVecs = 2;  // of a sub-key row: (dq/2)*esz <= 1 KiB
constexpr int kDecodeKeys = kSChunk / kSmallWarps;  // sub-keys per warp (8)
constexpr int kMmaMaxKB = 8;  // MMA tiles: 32-wide K-blocks of a sub-key row in registers

// bf16 layers whose query network and per-half scores can run as the tensor-core tiles
// below (d_model and dq/2 multiples of 32, dq/2 <= 256).
__host__ __device__ inline bool mma_shape(int d, int dq, int esz) {
  const int half = dq / 2;
  return esz == 2 && d % 32 == 0 && half % 32 == 0 && half <= 32 * kMmaMaxKB;
}

// Largest batch decode mode takes. Where the tensor-core tiles can run instead they
// measured faster from 6 tokens with H = 4 (1024^2 layer, us per call: 12.4 vs 16.3 for
// one token, 15.8 vs 17.3 for 4, 18.9 vs 18.2 for 6, 21.8 vs 19.5 for 8) and from one
// token with H = 8 (wide layer: 20.7 vs 19.9 for one, 29.6 vs 20.5 for 4): decode mode's
// warps take the tokens one after another.
__host__ __device__ inline int decode_max_b(int H, int d, int dq, int esz) {
  if (!mma_shape(d, dq, esz)) return kDecodeB;
  return H <= 4 ? 4 : 0;
}

__host__ __device__ inline bool decode_mode(int64_t B, int H, int d, int dq, int esz) {
  const int rb = d * esz, kb = (dq / 2) * esz;
  return B >= 1 && B <= decode_max_b(H, d, dq, esz) && rb % 16 == 0 && kb % 16 == 0 &&
         rb <= 16 * 32 * kDecodeRowVecs && kb <= 16 * 32 * kDecodeKeyVecs;
}

__device__ __forceinline__ float xor_tree_sum(float p) {
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) p += __shfl_xor_sync(0xffffffffu, p, m);
  return p;
}

// q[t][f] for every token t < B (one warp): W_q row f against each token's x row, then
// the BatchNorm affine map as in the kernels below.
template <typename T, int RV>
__device__ __forceinline__ void decode_query_row(const T* __restrict__ x, const T* __restrict__ W,
                                                 const float* __restrict__ mean,
                                                 const float* __restrict__ var,
                                                 const float* __restrict__ gamma,
                                                 const float* __restrict__ beta, float eps,
                                                 int B, int d, int F, int f,
                                                 float* __restrict__ q) {
  constexpr int VPER = Vec<T>::kPer;
  const int lane = threadIdx.x & 31;
  const int nch = d / VPER;  // 16-byte chunks per row
  const uint4* wr = reinterpret_cast<const uint4*>(W + static_cast<int64_t>(f) * d);
  uint4 wv[RV];
#pragma unroll
  for (int i = 0; i < RV; ++i) {
    const int c = lane + 32 * i;
    wv[i] = c < nch ? __ldg(wr + c) : make_uint4(0, 0, 0, 0);
  }
  float sc = 0.f, sh = 0.f;
  if (lane == 0) {
    sc = gamma[f] / sqrtf(var[f] + eps);
    sh = beta[f] - mean[f] * sc;
  }
  // Two tokens at a time, so that both x rows' loads are in flight together.
  for (int t = 0; t < B; t += 2) {
    const bool two = t + 1 < B;  // warp-uniform
    const uint4* xr0 = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d);
    const uint4* xr1 = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t + 1) * d);
    uint4 xv0[RV], xv1[RV];
#pragma unroll
    for (int i = 0; i < RV; ++i) {
      const int c = lane + 32 * i;
      xv0[i] = c < nch ? __ldg(xr0 + c) : make_uint4(0, 0, 0, 0);
      xv1[i] = (two && c < nch) ? __ldg(xr1 + c) : make_uint4(0, 0, 0, 0);
    }
    float p0 = 0.f, p1 = 0.f;
#pragma unroll
    for (int i = 0; i < RV; ++i) {
      if (lane + 32 * i < nch) {
        float x0[VPER], x1[VPER], wf[VPER];
        Vec<T>::widen(xv0[i], x0);
        Vec<T>::widen(xv1[i], x1);
        Vec<T>::widen(wv[i], wf);
#pragma unroll
        for (int e = 0; e < VPER; ++e) {
          p0 = fmaf(x0[e], wf[e], p0);
          p1 = fmaf(x1[e], wf[e], p1);
        }
      }
    }
    p0 = xor_tree_sum(p0);
    p1 = xor_tree_sum(p1);
    if (lane == 0) {
      q[static_cast<int64_t>(t) * F + f] = fmaf(p0, sc, sh);
      if (two) q[static_cast<int64_t>(t + 1) * F + f] = fmaf(p1, sc, sh);
    }
  }
}

// This warp's kDecodeKeys sub-key rows c0 + kDecodeKeys * warp + r of head-half hs
// (rows past n read as zeros).
template <typename T, int KV>
__device__ __forceinline__ void decode_load_keys(const T* __restrict__ C, int n, int half, int hs,
                                                 int c0, uint4 (&kv)[kDecodeKeys][KV]) {
  constexpr int VPER = Vec<T>::kPer;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = half / VPER;
#pragma unroll
  for (int r = 0; r < kDecodeKeys; ++r) {
    const int c = c0 + kDecodeKeys * warp + r;
    const uint4* kr = reinterpret_cast<const uint4*>(C + (static_cast<int64_t>(hs) * n + c) * half);
#pragma unroll
    for (int i = 0; i < KV; ++i) {
      const int ch = lane + 32 * i;
      kv[r][i] = (c < n && ch < nch) ? __ldg(kr + ch) : make_uint4(0, 0, 0, 0);
    }
  }
}

// Scores of those rows against each token's query half (fp32, from global memory),
// written to sc[t][kDecodeKeys * warp + r] (kSChunk floats per token).
template <typename T, int KV>
__device__ __forceinline__ void decode_score_keys(const float* __restrict__ q, int B, int F,
                                                  int dq, int hs, const uint4 (&kv)[kDecodeKeys][KV],
                                                  float* sc) {
  constexpr int VPER = Vec<T>::kPer;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = dq >> 1;
  const int nch = half / VPER;
  const int off = (hs >> 1) * dq + (hs & 1) * half;
  for (int t = 0; t < B; ++t) {
    const float* qt = q + static_cast<int64_t>(t) * F + off;
    float qf[KV][VPER];
#pragma unroll
    for (int i = 0; i < KV; ++i) {
      const int ch = lane + 32 * i;
#pragma unroll
      for (int e = 0; e < VPER; e += 4) {
        const float4 v4 = ch < nch ? __ldcg(reinterpret_cast<const float4*>(qt + ch * VPER + e))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        qf[i][e] = v4.x;
        qf[i][e + 1] = v4.y;
        qf[i][e + 2] = v4.z;
        qf[i][e + 3] = v4.w;
      }
    }
    float p[kDecodeKeys];
#pragma unroll
    for (int r = 0; r < kDecodeKeys; ++r) {
      p[r] = 0.f;
#pragma unroll
      for (int i = 0; i < KV; ++i) {
        if (lane + 32 * i < nch) {
          float kf[VPER];
          Vec<T>::widen(kv[r][i], kf);
#pragma unroll
          for (int e = 0; e < VPER; ++e) p[r] = fmaf(qf[i][e], kf[e], p[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kDecodeKeys; ++r) p[r] = xor_tree_sum(p[r]);
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < kDecodeKeys; ++r) sc[t * kSChunk + kDecodeKeys * warp + r] = p[r];
    }
  }
}

// Token t's best 32 of the chunk's kSChunk scores (one warp; rows past n excluded), in
// the order the kernels below write chunk lists.
__device__ __forceinline__ void decode_chunk_list(const float* sc, int t, int c0, int n,
                                                  float& s0, int& i0) {
  const int lane = threadIdx.x & 31;
  const bool v0 = c0 + lane < n, v1 = c0 + 32 + lane < n;
  s0 = v0 ? sc[t * kSChunk + lane] : -INFINITY;
  float s1 = v1 ? sc[t * kSChunk + 32 + lane] : -INFINITY;
  i0 = v0 ? c0 + lane : kIdPad;
  int i1 = v1 ? c0 + 32 + lane : kIdPad;
  warp_sort32(s0, i0);
  warp_sort32(s1, i1);
  warp_merge32(s0, i0, s1, i1);
}

// ---------------------------------------------------------------------------
// bf16 layers past decode mode: the query network and the per-half scores as
// warp-level tensor-core products (mma.sync m16n8k16: bf16 operands, fp32
// accumulation) on tiles of kMmaTok tokens, used by both small-batch forms.
//
// The operands go from global memory straight into the MMA fragments. A contraction
// may run over its index in any order as long as both operands use the same one:
// thread (g = lane / 4, t = lane % 4) of an MMA holds, for rows g and g + 8 of A and
// column g of B, the k in {2t, 2t+1, 2t+8, 2t+9}; here those are the elements
// 8t .. 8t+3 of a 32-wide K-block for the block's first MMA and 8t+4 .. 8t+7 for its
// second, so a thread reads its 8 elements of a row as one 16-byte load.
//
// q stays an fp32 result ("Large Memory Layers with Product Keys", gptget.net summary,
// Methodology: the query network is a linear map followed by batch normalisation):
// the query tile accumulates x W_q^T in fp32, and the score tile splits q into
// hi = RN_bf16(q) and lo = RN_bf16(q - hi) (residual at most 2^-16 |q|) with one fp32
// accumulator per plane; sub-keys are bf16 and exact.
// ---------------------------------------------------------------------------
constexpr int kMmaTok = 16;     // tokens per tile (the MMA's M)
constexpr int kMmaFeat = 16;    // features per query tile (two 8-wide MMA N tiles)
constexpr int kMmaKSplit = kSmallWarps / 2;  // query tile: warps sharing an N tile's K
constexpr int kMmaRedLd = kMmaFeat + 1;

__host__ __device__ inline bool mma_mode(int64_t B, int H, int d, int dq, int esz) {
  return mma_shape(d, dq, esz) && !decode_mode(B, H, d, dq, esz);
}

// Shared memory of the query tile: the K-split partial sums [kMmaKSplit][16][17].
constexpr size_t kMmaQuerySmem = sizeof(float) * kMmaKSplit * kMmaTok * kMmaRedLd;

// Shared memory of the score tile: q of its tokens as bf16 planes hi and lo,
// [2][16][half + 32] (64 bytes of padding per row keep the fragment reads free of bank
// conflicts), then the scores [16][kSChunk].
__host__ __device__ inline size_t mma_score_smem(int half) {
  return static_cast<size_t>(2) * kMmaTok * (half + 32) * 2 +
         sizeof(float) * kMmaTok * kSChunk;
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The two MMAs of a 32-wide K-block: this thread's pieces of A rows g (ra) and g + 8
// (rb) and of B column g (bv).
__device__ __forceinline__ void mma_kblock(float (&c)[4], const uint4& ra, const uint4& rb,
                                           const uint4& bv) {
  mma16816(c, ra.x, rb.x, ra.y, rb.y, bv.x, bv.y);
  mma16816(c, ra.z, rb.z, ra.w, rb.w, bv.z, bv.w);
}

// hi = RN_bf16(q), lo = RN_bf16(q - hi) of two consecutive elements, packed in pairs.
__device__ __forceinline__ void split2_pair(float q0, float q1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(q0, q1);
  const __nv_bfloat162 l = __floats2bfloat162_rn(q0 - __low2float(h), q1 - __high2float(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// q[t0 .. t0+15][f0 .. f0+15] = BN(x W_q^T) for the tokens below B (one CTA of 8 warps;
// F is a multiple of 16). Warp w takes the 8 features f0 + 8 (w % 2) + [0, 8) over the
// K-blocks kb = w / 2 (mod kMmaKSplit); the partial products of a feature are added in
// K-split order through shared memory (red, kMmaQuerySmem bytes), then the BatchNorm
// affine map as in the kernels above.
__device__ void mma_query_tile(const uint16_t* __restrict__ X, const uint16_t* __restrict__ W,
                               const float* __restrict__ mean, const float* __restrict__ var,
                               const float* __restrict__ gamma, const float* __restrict__ beta,
                               float eps, int B, int d, int F, int f0, int t0, float* red,
                               float* __restrict__ q) {
  constexpr int U = 4;  // K-blocks in flight per thread
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nt = warp & 1, ks = warp >> 1;
  const int nkb = d >> 5;
  const int ra = t0 + g, rb = t0 + g + 8;
  const bool oka = ra < B, okb = rb < B;
  const uint4 z = make_uint4(0, 0, 0, 0);
  const uint4* xa = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(oka ? ra : 0) * d) + t;
  const uint4* xb = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(okb ? rb : 0) * d) + t;
  const uint4* wr = reinterpret_cast<const uint4*>(W + static_cast<int64_t>(f0 + 8 * nt + g) * d) + t;
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  for (int kb0 = ks; kb0 < nkb; kb0 += U * kMmaKSplit) {
    uint4 pa[U], pb[U], pw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int kb = kb0 + u * kMmaKSplit;
      const bool live = kb < nkb;
      pa[u] = live && oka ? __ldg(xa + 4 * kb) : z;
      pb[u] = live && okb ? __ldg(xb + 4 * kb) : z;
      pw[u] = live ? __ldg(wr + 4 * kb) : z;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) mma_kblock(c, pa[u], pb[u], pw[u]);
  }
  float* rp = red + ks * kMmaTok * kMmaRedLd;
  const int col = 8 * nt + 2 * t;
  rp[g * kMmaRedLd + col] = c[0];
  rp[g * kMmaRedLd + col + 1] = c[1];
  rp[(g + 8) * kMmaRedLd + col] = c[2];
  rp[(g + 8) * kMmaRedLd + col + 1] = c[3];
  __syncthreads();
  const int row = threadIdx.x / kMmaFeat, fc = threadIdx.x % kMmaFeat;  // 256 = 16 x 16
  const int tok = t0 + row, f = f0 + fc;
  if (tok < B) {
    float s = red[row * kMmaRedLd + fc];
#pragma unroll
    for (int i = 1; i < kMmaKSplit; ++i) s += red[(i * kMmaTok + row) * kMmaRedLd + fc];
    const float sc = gamma[f] / sqrtf(var[f] + eps);
    q[static_cast<int64_t>(tok) * F + f] = fmaf(s, sc, beta[f] - mean[f] * sc);
  }
  __syncthreads();  // red is free again
}

// This warp's B fragments of a score tile: sub-keys c0 + 8 warp + g of head-half hs,
// piece t of each 32-wide K-block (sub-keys past n read as zeros).
__device__ __forceinline__ void mma_load_keys(const uint16_t* __restrict__ C, int n, int half,
                                              int hs, int c0, uint4 (&kf)[kMmaMaxKB]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int key = c0 + 8 * warp + (lane >> 2);
  const bool ok = key < n;
  const uint4* src = reinterpret_cast<const uint4*>(
                         C + (static_cast<int64_t>(hs) * n + (ok ? key : 0)) * half) + (lane & 3);
  const int nkb = half >> 5;
#pragma unroll
  for (int kb = 0; kb < kMmaMaxKB; ++kb)
    kf[kb] = ok && kb < nkb ? __ldg(src + 4 * kb) : make_uint4(0, 0, 0, 0);
}

// Scores of the sub-keys c0 .. c0+63 of head-half hs (kf from mma_load_keys) against
// the query halves of tokens t0 .. t0+15 below B, and each token's best 32 of them
// into the chunk lists, as score_small_kernel writes them (one CTA of 8 warps; smem:
// mma_score_smem(dq / 2) bytes, 16-byte aligned). q is read through L2 (__ldcg): in
// the single-kernel form other CTAs wrote it during the same launch.
__device__ void mma_score_tile(const float* q, const uint4 (&kf)[kMmaMaxKB], int B, int H,
                               int dq, int n, int hs, int chunk, int t0, unsigned char* smem,
                               float* __restrict__ cs, int* __restrict__ ci) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int half = dq >> 1, F = H * dq;
  const int h = hs >> 1, side = hs & 1;
  const int ld = half + 32;  // elements per plane row
  uint16_t* qh = reinterpret_cast<uint16_t*>(smem);
  uint16_t* ql = qh + kMmaTok * ld;
  float* sc = reinterpret_cast<float*>(ql + kMmaTok * ld);  // [16][kSChunk]
  const int c0 = chunk * kSChunk;
  const int nchunks = (n + kSChunk - 1) / kSChunk;
  __syncthreads();  // the previous tile has finished with the shared memory
  const int per_row = half >> 2;  // float4 per query half
  for (int i = threadIdx.x; i < kMmaTok * per_row; i += blockDim.x) {
    const int r = i / per_row, e = (i - r * per_row) * 4;
    const int tok = t0 + r;
    const float4 v = tok < B ? __ldcg(reinterpret_cast<const float4*>(
                                   q + static_cast<int64_t>(tok) * F + h * dq + side * half + e))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    uint32_t h0, l0, h1, l1;
    split2_pair(v.x, v.y, h0, l0);
    split2_pair(v.z, v.w, h1, l1);
    *reinterpret_cast<uint2*>(qh + r * ld + e) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(ql + r * ld + e) = make_uint2(l0, l1);
  }
  __syncthreads();
  float chi[4] = {0.f, 0.f, 0.f, 0.f}, clo[4] = {0.f, 0.f, 0.f, 0.f};
  const int nkb = half >> 5;
#pragma unroll
  for (int kb = 0; kb < kMmaMaxKB; ++kb) {
    if (kb < nkb) {
      const int e = kb * 32 + 8 * t;
      const uint4 ha = *reinterpret_cast<const uint4*>(qh + g * ld + e);
      const uint4 hb = *reinterpret_cast<const uint4*>(qh + (g + 8) * ld + e);
      const uint4 la = *reinterpret_cast<const uint4*>(ql + g * ld + e);
      const uint4 lb = *reinterpret_cast<const uint4*>(ql + (g + 8) * ld + e);
      mma_kblock(chi, ha, hb, kf[kb]);
      mma_kblock(clo, la, lb, kf[kb]);
    }
  }
  const int col = 8 * warp + 2 * t;
  *reinterpret_cast<float2*>(sc + g * kSChunk + col) = make_float2(chi[0] + clo[0], chi[1] + clo[1]);
  *reinterpret_cast<float2*>(sc + (g + 8) * kSChunk + col) =
      make_float2(chi[2] + clo[2], chi[3] + clo[3]);
  __syncthreads();
  // Warp w selects for the tile's tokens w and w + 8.
  for (int r = warp; r < kMmaTok; r += kSmallWarps) {
    const int tok = t0 + r;
    if (tok >= B) break;  // warp-uniform
    float s0;
    int i0;
    decode_chunk_list(sc, r, c0, n, s0, i0);
    const int64_t o =
        ((((static_cast<int64_t>(tok) * H + h) * 2 + side) * nchunks + chunk) << 5) + lane;
    cs[o] = s0;
    ci[o] = i0;
  }
}

// The three-kernel form's query and scoring kernels in that mode: CTA = (16 features,
// 16 tokens) and CTA = (64 sub-keys, head-half, 16 tokens).
__global__ void __launch_bounds__(kSmallWarps * 32) query_mma_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ W,
    const float* __restrict__ mean, const float* __restrict__ var,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps, int B, int d,
    int F, float* __restrict__ q, int* clear) {
  __shared__ float red[kMmaKSplit * kMmaTok * kMmaRedLd];
  first_kernel_prologue(clear);
  mma_query_tile(x, W, mean, var, gamma, beta, eps, B, d, F, blockIdx.x * kMmaFeat,
                 blockIdx.y * kMmaTok, red, q);
}

__global__ void __launch_bounds__(kSmallWarps * 32, 4) score_mma_kernel(
    const float* __restrict__ q, const uint16_t* __restrict__ subkeys, int B, int H, int dq,
    int n, float* __restrict__ chunk_s, int* __restrict__ chunk_i) {
  extern __shared__ __align__(16) unsigned char sm_raw[];
  allow_dependents();
  uint4 kf[kMmaMaxKB];
  mma_load_keys(subkeys, n, dq / 2, blockIdx.y, blockIdx.x * kSChunk, kf);
  wait_prior_grid();  // q comes from the query kernel
  mma_score_tile(q, kf, B, H, dq, n, blockIdx.y, blockIdx.x, blockIdx.z * kMmaTok, sm_raw,
                 chunk_s, chunk_i);
}

// ---------------------------------------------------------------------------
// q[t][f] = (sum_c x[t][c] W[f][c]) * scale[f] + shift[f], scale = gamma / sqrt(var + eps),
// shift = beta - mean * scale (the tensor-core epilogue's form). CTA = 16 features x 8
// tokens: the 16 rows of W_q and the 8 rows of x staged in shared memory, one warp
// per token, each lane reading bf16 rows two elements (one 32-bit word) at a time,
// 4 words in flight; the 16 per-lane partial sums are reduced by a butterfly that
// leaves feature j's total in lanes 2j and 2j + 1 (16 shuffles instead of 80).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kSmallWarps * 32) query_small_kernel(
    const T* __restrict__ x, const T* __restrict__ W, const float* __restrict__ mean,
    const float* __restrict__ var, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, int B, int d, int F, float* __restrict__ q,
    int* clear) {
  extern __shared__ __align__(16) unsigned char qs_raw[];
  T* ws = reinterpret_cast<T*>(qs_raw);  // [kQFeat][d]
  T* xs = ws + kQFeat * d;               // [kQTok][d]
  first_kernel_prologue(clear);
  const int f0 = blockIdx.x * kQFeat;
  const int nf = min(kQFeat, F - f0);
  const int t0 = blockIdx.y * kQTok;
  // d * sizeof(T) is a multiple of 4 (checked on the host): whole rows are words.
  const int row_words = d * static_cast<int>(sizeof(T)) / 4;
  stage_rows(reinterpret_cast<const uint32_t*>(W + static_cast<int64_t>(f0) * d),
             reinterpret_cast<uint32_t*>(ws), kQFeat, nf, row_words, row_words);
  stage_rows(reinterpret_cast<const uint32_t*>(x + static_cast<int64_t>(t0) * d),
             reinterpret_cast<uint32_t*>(xs), kQTok, min(kQTok, B - t0), row_words, row_words);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = t0 + warp;
  if (t < B) {
    float acc[kQFeat];
#pragma unroll
    for (int j = 0; j < kQFeat; ++j) acc[j] = 0.f;
    const T* xr = xs + warp * d;
    if constexpr (sizeof(T) == 2) {
      // bf16: one 32-bit shared-memory word holds two consecutive columns (d is even).
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(xr);
      const uint32_t* ww = reinterpret_cast<const uint32_t*>(ws);
      const int dw = d >> 1;
      for (int c0 = 0; c0 < dw; c0 += 32 * 4) {
        uint32_t xv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + lane + 32 * u;
          xv[u] = c < dw ? xw[c] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + lane + 32 * u;
          if (c < dw) {
            const float xa = bf16_lo(xv[u]), xb = bf16_hi(xv[u]);
#pragma unroll
            for (int j = 0; j < kQFeat; ++j) {
              const uint32_t wv = ww[j * dw + c];
              acc[j] = fmaf(xb, bf16_hi(wv), fmaf(xa, bf16_lo(wv), acc[j]));
            }
          }
        }
      }
    } else {
      for (int c0 = 0; c0 < d; c0 += 32 * 8) {
        float xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + lane + 32 * u;
          xv[u] = c < d ? load_elem(xr, c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + lane + 32 * u;
          if (c < d) {
#pragma unroll
            for (int j = 0; j < kQFeat; ++j) acc[j] = fmaf(xv[u], load_elem(ws, j * d + c), acc[j]);
          }
        }
      }
    }
    // Butterfly: at mask m each lane keeps half of its values (the upper half when
    // its bit m is set) and adds the partner's copy of them.
#pragma unroll
    for (int m = 16, c = kQFeat / 2; c >= 1; m >>= 1, c >>= 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < c; ++i) {
        const float send = up ? acc[i] : acc[i + c];
        const float keep = up ? acc[i + c] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
    const float a = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
    const int j = lane >> 1;  // this lane's feature
    if ((lane & 1) == 0 && j < nf) {
      const int f = f0 + j;
      const float sc = gamma[f] / sqrtf(var[f] + eps);
      q[static_cast<int64_t>(t) * F + f] = fmaf(a, sc, beta[f] - mean[f] * sc);
    }
  }
}

// ---------------------------------------------------------------------------
// Per-half scores of one chunk of kSChunk sub-keys for up to kSTok tokens, and each
// token's best 32 of the chunk. Lane i scores sub-keys c0 + i and c0 + 32 + i (a
// 32-bit word, two elements, of each bf16 row per step); the two
// sorted halves are merged (warp_sort32 / warp_merge32). Output chunk lists
// [B][H][2][nchunks][32], best first (padding: -inf, kIdPad).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kSmallWarps * 32) score_small_kernel(
    const float* __restrict__ q, const T* __restrict__ subkeys, int B, int H, int dq, int n,
    float* __restrict__ chunk_s, int* __restrict__ chunk_i) {
  extern __shared__ __align__(16) unsigned char ss_raw[];
  const int half = dq >> 1;
  const int ld = half + (sizeof(T) == 2 ? 2 : 1);  // padded row: lanes hit distinct banks
  T* rows = reinterpret_cast<T*>(ss_raw);           // [kSChunk][ld]
  float* qs = reinterpret_cast<float*>(ss_raw + ((sizeof(T) * kSChunk * ld + 15) & ~15));
  const int chunk = blockIdx.x, hs = blockIdx.y;
  const int h = hs >> 1, side = hs & 1;
  const int c0 = chunk * kSChunk;
  const int nchunks = (n + kSChunk - 1) / kSChunk;
  const T* book = subkeys + (static_cast<int64_t>(hs) * n + c0) * half;
  // half * sizeof(T) is a multiple of 4 (checked on the host); ld * sizeof(T) too.
  const int row_words = half * static_cast<int>(sizeof(T)) / 4;
  allow_dependents();
  stage_rows(reinterpret_cast<const uint32_t*>(book), reinterpret_cast<uint32_t*>(rows),
             kSChunk, min(kSChunk, n - c0), row_words, ld * static_cast<int>(sizeof(T)) / 4);
  wait_prior_grid();  // q comes from the query kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int F = H * dq;
  // The warp's two tokens' query halves.
  float* qw = qs + warp * 2 * half;
  const int tb = blockIdx.z * kSTok + warp * 2;
  for (int i0 = 0; i0 < 2 * half; i0 += 32 * 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + lane + 32 * u;
      const int uu = i / half, e = i - uu * half;
      const int t = tb + uu;
      v[u] = (i < 2 * half && t < B) ? q[static_cast<int64_t>(t) * F + h * dq + side * half + e]
                                     : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + lane + 32 * u;
      if (i < 2 * half) qw[i] = v[u];
    }
  }
  __syncthreads();
  const bool v0 = c0 + lane < n, v1 = c0 + 32 + lane < n;
  const T* r0 = rows + lane * ld;
  const T* r1 = rows + (lane + 32) * ld;
  for (int u = 0; u < 2; ++u) {
    const int t = tb + u;
    if (t >= B) break;  // warp-uniform
    const float* qq = qw + u * half;
    // Two chains per row (even and odd elements), added at the end. half is even; a
    // bf16 row is read a 32-bit word (two elements) at a time.
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    for (int e = 0; e < half; e += 2) {
      const float2 qv = *reinterpret_cast<const float2*>(qq + e);
      float x0a, x0b, x1a, x1b;
      if constexpr (sizeof(T) == 2) {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(r0 + e);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(r1 + e);
        x0a = bf16_lo(w0); x0b = bf16_hi(w0);
        x1a = bf16_lo(w1); x1b = bf16_hi(w1);
      } else {
        x0a = load_elem(r0, e); x0b = load_elem(r0, e + 1);
        x1a = load_elem(r1, e); x1b = load_elem(r1, e + 1);
      }
      a0 = fmaf(qv.x, x0a, a0);
      a1 = fmaf(qv.x, x1a, a1);
      b0 = fmaf(qv.y, x0b, b0);
      b1 = fmaf(qv.y, x1b, b1);
    }
    a0 += b0;
    a1 += b1;
    float s0 = v0 ? a0 : -INFINITY, s1 = v1 ? a1 : -INFINITY;
    int i0 = v0 ? c0 + lane : kIdPad, i1 = v1 ? c0 + 32 + lane : kIdPad;
    warp_sort32(s0, i0);
    warp_sort32(s1, i1);
    warp_merge32(s0, i0, s1, i1);
    const int64_t o = ((((static_cast<int64_t>(t) * H + h) * 2 + side) * nchunks + chunk) << 5) + lane;
    chunk_s[o] = s0;
    chunk_i[o] = i0;
  }
}

// ---------------------------------------------------------------------------
// Decode mode of the three-kernel form (at most kDecodeB tokens): the two kernels
// above with a warp per W_q row / per kDecodeKeys sub-keys instead of per token. Kept
// apart from them so that their register budgets stay small.
// ---------------------------------------------------------------------------
template <typename T, int RV>
__global__ void __launch_bounds__(kSmallWarps * 32) query_decode_kernel(
    const T* __restrict__ x, const T* __restrict__ W, const float* __restrict__ mean,
    const float* __restrict__ var, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, int B, int d, int F, float* __restrict__ q,
    int* clear) {
  first_kernel_prologue(clear);
  const int f = blockIdx.x * kSmallWarps + (threadIdx.x >> 5);
  if (f < F) decode_query_row<T, RV>(x, W, mean, var, gamma, beta, eps, B, d, F, f, q);
}

// Grid (chunks, 2H): block = 64 sub-keys of one head-half for every token; warp t then
// writes token t's chunk list.
template <typename T, int KV>
__global__ void __launch_bounds__(kSmallWarps * 32) score_decode_kernel(
    const float* __restrict__ q, const T* __restrict__ subkeys, int B, int H, int dq, int n,
    float* __restrict__ chunk_s, int* __restrict__ chunk_i) {
  __shared__ float scs[kDecodeB * kSChunk];
  const int chunk = blockIdx.x, hs = blockIdx.y;
  const int h = hs >> 1, side = hs & 1;
  const int c0 = chunk * kSChunk;
  const int nchunks = (n + kSChunk - 1) / kSChunk;
  allow_dependents();
  uint4 kv[kDecodeKeys][KV];
  decode_load_keys<T, KV>(subkeys, n, dq >> 1, hs, c0, kv);
  wait_prior_grid();  // q comes from the query kernel
  decode_score_keys<T, KV>(q, B, H * dq, dq, hs, kv, scs);
  __syncthreads();
  const int t = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t < B) {
    float s0;
    int i0;
    decode_chunk_list(scs, t, c0, n, s0, i0);
    const int64_t o =
        ((((static_cast<int64_t>(t) * H + h) * 2 + side) * nchunks + chunk) << 5) + lane;
    chunk_s[o] = s0;
    chunk_i[o] = i0;
  }
}

// ---------------------------------------------------------------------------
// One CTA per (token, head); the H CTAs of a token form a thread-block cluster.
// (a) The chunk lists of the head's two halves merged into each half's best 32, four
// lists per warp in registers, then a tree over the warps. (b) Exact top-k of the
// pruned product candidates (sorted 32 per warp, tree-merged), then warp 0: softmax,
// indices / weights / scores. (c) The k weighted value rows, split over the 8 warps,
// added in warp order. (d) Each CTA owns a slice of the columns of out[t]: every CTA
// stores its head's sums of each slice into the owner's shared memory (distributed
// shared memory), one cluster barrier, then each owner adds the H rows of its slice in
// head order and writes them. The cluster barrier is split: arrived at at the start
// (relaxed), waited for before the first store into another CTA, so its wait only
// confirms that every CTA of the cluster is running.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");  // release
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // acquire
}

// Floats of the head-sum receive buffer: H slices of ceil(v / H) columns (H <= 8).
__host__ __device__ inline int gather_part_len(int v) { return (v + 8 + 3) & ~3; }

// MINB: CTAs per SM the register budget is sized for (the launch picks 4 when a grid of
// (token, head) CTAs would not fit on the GPU at once with the default budget).
template <typename T, int MAXV, int MINB>
__global__ void __launch_bounds__(kSmallWarps * 32, MINB) gather_small_kernel(
    const float* __restrict__ chunk_s, const int* __restrict__ chunk_i,
    const T* __restrict__ values, int H, int n, int k, int v, float* __restrict__ out,
    int* __restrict__ indices, float* __restrict__ weights, float* __restrict__ scores,
    int* status) {
  namespace cg = cooperative_groups;
  constexpr int VPER = Vec<T>::kPer;
  extern __shared__ __align__(16) unsigned char gs_raw[];
  const int nchunks = (n + kSChunk - 1) / kSChunk;
  const int list_words = 2 * nchunks * kMaxK;                    // this head's two halves
  float* part = reinterpret_cast<float*>(gs_raw);  // [H][v / H] received head sums
  float* red = part + gather_part_len(v);           // [kSmallWarps][v]
  float* cls = red;                                               // [2][nchunks][32] (phase a)
  int* cli = reinterpret_cast<int*>(red + list_words);
  const int scratch = max(kSmallWarps * v, 2 * list_words);
  float* cand_s = red + scratch;                                  // [kMaxPairs]
  int* cand_i = reinterpret_cast<int*>(cand_s + kMaxPairs);       // [kMaxPairs]
  int* rows = cand_i + kMaxPairs;                                 // [k]
  float* wts = reinterpret_cast<float*>(rows + kMaxK);            // [k]
  int* pairs = reinterpret_cast<int*>(wts + kMaxK);               // [kMaxPairs]
  __shared__ int npairs_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t = blockIdx.x;
  const int h = blockIdx.y;  // also the CTA's rank in its cluster
  cluster_arrive_relaxed();
  if (threadIdx.x == 0) npairs_s = build_pairs(k, pairs);
  wait_prior_grid();  // the chunk lists come from the scoring kernel
  // The stream's next kernel may launch now: a later call's first kernel waits for this
  // grid's end before it reads anything.
  allow_dependents();
  const int64_t src = (t * H + h) * list_words;

  // (a) each half's best 32. Warp w takes up to 4 of a half's chunk lists straight into
  // registers (lane j holding entry j of each) and merges them, two merges side by side
  // and then one; the warps' lists (4 per half on the 1024^2 layer) are then merged as a
  // tree in shared memory: at stride st the list at 2 st i + st into the list at 2 st i.
  const int quads = (nchunks + 3) / 4;  // warp lists per half
  for (int item = warp; item < 2 * quads; item += kSmallWarps) {
    const int side = item / quads, qd = item - side * quads;
    const int nl = min(4, nchunks - 4 * qd);
    const int64_t g0 = src + ((side * nchunks + 4 * qd) << 5) + lane;
    float ls4[4];
    int li4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      ls4[u] = u < nl ? __ldg(chunk_s + g0 + 32 * u) : -INFINITY;
      li4[u] = u < nl ? __ldg(chunk_i + g0 + 32 * u) : kIdPad;
    }
    warp_merge32(ls4[0], li4[0], ls4[1], li4[1]);
    warp_merge32(ls4[2], li4[2], ls4[3], li4[3]);
    warp_merge32(ls4[0], li4[0], ls4[2], li4[2]);
    cls[((side * quads + qd) << 5) + lane] = ls4[0];
    cli[((side * quads + qd) << 5) + lane] = li4[0];
  }
  __syncthreads();
  for (int st = 1; st < quads; st <<= 1) {
    const int per_side = (quads + 2 * st - 1) / (2 * st);
    for (int item = warp; item < 2 * per_side; item += kSmallWarps) {
      const int side = item / per_side, i = item - side * per_side;
      const int a0 = 2 * st * i, b0 = a0 + st;
      if (b0 >= quads) continue;  // warp-uniform
      const int pa = ((side * quads + a0) << 5) + lane, pb = ((side * quads + b0) << 5) + lane;
      float bs = cls[pa];
      int bi = cli[pa];
      warp_merge32(bs, bi, cls[pb], cli[pb]);
      cls[pa] = bs;
      cli[pa] = bi;
    }
    __syncthreads();
  }
  float* ls = cls;                          // half 0's best 32 at list 0, half 1's after
  int* li = cli;
  const int l1 = quads << 5;

  // (b) the pruned candidates in chunks of 32, one chunk per warp, each sorted; then
  // merged as a tree; warp 0 takes softmax and the head's picks.
  const int npairs = npairs_s;
  const int nc = (npairs + 31) / 32;
  for (int c = warp; c < nc; c += kSmallWarps) {
    const int p = c * 32 + lane;
    const int ab = p < npairs ? pairs[p] : 0;
    const int pa = ab & 0xff, pb = ab >> 8;
    const float sa = ls[pa], sb = ls[l1 + pb];
    const int ia = li[pa], ib = li[l1 + pb];
    // Padding ids can only surface when scores are NaN; they never form a slot.
    const bool real = p < npairs && ia >= 0 && ia < n && ib >= 0 && ib < n;
    float cs = real ? sa + sb : -INFINITY;
    int ci = real ? ia * n + ib : kIdPad;
    warp_sort32(cs, ci);
    cand_s[(c << 5) + lane] = cs;
    cand_i[(c << 5) + lane] = ci;
  }
  __syncthreads();
  for (int st = 1; st < nc; st <<= 1) {
    for (int i = warp; 2 * st * i + st < nc; i += kSmallWarps) {
      const int pa = ((2 * st * i) << 5) + lane, pb = ((2 * st * i + st) << 5) + lane;
      float bs = cand_s[pa];
      int bi = cand_i[pa];
      warp_merge32(bs, bi, cand_s[pb], cand_i[pb]);
      cand_s[pa] = bs;
      cand_i[pa] = bi;
    }
    __syncthreads();
  }
  if (warp == 0) {
    const float bs = cand_s[lane];
    const int bi = cand_i[lane];
    const float mx = __shfl_sync(0xffffffffu, bs, 0);
    const float e = lane < k ? expf(bs - mx) : 0.f;
    const float den = warp_sum(e);
    const float w = e / den;
    if (lane < k) {
      const int64_t o = (t * H + h) * static_cast<int64_t>(k) + lane;
      indices[o] = bi;
      weights[o] = w;
      if (scores) scores[o] = bs;
      rows[lane] = bi;
      wts[lane] = w;
    }
  }
  __syncthreads();

  // (c) weighted value rows r = warp, warp + 8, ... (all of a warp's rows in flight).
  constexpr int U = 4;  // k <= 32 rows over 8 warps
  const int nvec = v / VPER;
  float acc[MAXV][VPER];
#pragma unroll
  for (int m = 0; m < MAXV; ++m)
#pragma unroll
    for (int e = 0; e < VPER; ++e) acc[m][e] = 0.f;
  {
    uint4 raw[U][MAXV];
    float wr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = warp + u * kSmallWarps;
      bool live = r < k;
      int row = live ? rows[r] : 0;
      if (live && (row < 0 || row >= n * n)) {  // only reachable with NaN scores
        if (lane == 0) record_status(status, kDevBadSlot);
        live = false;
        row = 0;
      }
      wr[u] = live ? wts[r] : 0.f;
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
  float* my = red + warp * v;
#pragma unroll
  for (int m = 0; m < MAXV; ++m) {
    const int vec = lane + 32 * m;
    if (vec < nvec) {
#pragma unroll
      for (int e = 0; e < VPER; ++e) my[vec * VPER + e] = acc[m][e];
    }
  }
  __syncthreads();
  // (d) this head's sum of column c goes to row h of the owner's receive buffer.
  cg::cluster_group cluster = cg::this_cluster();
  const int slice = (v + H - 1) / H;
  cluster_wait();  // every CTA of the cluster has started
  for (int c = threadIdx.x; c < v; c += blockDim.x) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < kSmallWarps; ++w) sum += red[w * v + c];
    const int owner = c / slice;
    cluster.map_shared_rank(part, owner)[h * slice + (c - owner * slice)] = sum;
  }
  cluster_arrive();  // this CTA's stores are done ...
  cluster_wait();    // ... and every other CTA's: the slice is complete
  const int c1 = min(v, (h + 1) * slice);
  for (int c = h * slice + threadIdx.x; c < c1; c += blockDim.x) {
    const int j = c - h * slice;
    float sum = part[j];
    for (int hh = 1; hh < H; ++hh) sum += part[hh * slice + j];
    out[t * v + c] = sum;
  }
}

// ---------------------------------------------------------------------------
// The same forward as ONE cooperative launch (one CTA per SM), its phases separated by
// grid-wide barriers instead of kernel boundaries:
//   Q  query network: in decode mode a warp per W_q row; with the tensor-core tiles
//      CTA = (16 features, 16 tokens) tiles; otherwise CTA = a group of 16 features
//      for all tokens (W_q rows staged once). Meanwhile the sub-keys of the CTA's
//      first scoring unit are prefetched into L2, since they do not depend on q
//   S  scores: CTA = (head-half, 64 sub-keys): scores for every token (the tiles:
//      the sub-keys held in registers across the 16-token tiles) and each token's best
//      32 of the chunk
//   G  gather: CTA = (token, head): the chunk lists merged per half (a tree over the
//      8 warps), exact top-k of the pruned candidates and softmax, the head's k
//      weighted value rows over 8 warps (all in flight), added in warp order into the
//      head's row of a workspace array; the token's last head to finish (a per-token
//      count) adds the H rows in head order into out
// A barrier is a counter in the workspace (zeroed by the host before the launch): each
// CTA adds one and waits, bounded by the pipelines' wait limit, until every CTA has; on
// a timeout the kernel records it in the status word and returns. Q and S use the same
// device functions and the same mode choice as the three-kernel form above, so picks,
// weights and scores are equal bit for bit; out adds each head's rows in the same
// order, heads in head order.
// ---------------------------------------------------------------------------
struct FusedArgs {
  const void* x;
  const void* W;
  const float* mean;
  const float* var;
  const float* gamma;
  const float* beta;
  const void* subkeys;
  const void* values;
  float eps;
  int B, d, H, dq, n, k, v;
  int decode;      // decode_mode(B, H, d, dq, esz)
  int mma;         // mma_mode(B, H, d, dq, esz)
  float* q;        // [B][H*dq] fp32
  float* cs;       // [B][H][2][nchunks][32] chunk lists
  int* ci;
  float* part;     // [B][H][v] each head's output row
  unsigned* tok_done;  // [B] heads of the token finished (phase G)
  float* out;
  int* idx;
  float* w;
  float* sc;
  int* status;
  unsigned* barrier;
};

// Returns false (every thread of the CTA) once the wait limit has passed.
__device__ bool fused_grid_sync(unsigned* counter, unsigned target, int* status, int* ok_s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(counter, 1u);
    unsigned seen;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(counter) : "memory");
    if (seen < target) {
      const uint64_t t0 = tc::global_timer_ns();
      for (;;) {
        __nanosleep(32);
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(counter) : "memory");
        if (seen >= target) break;
        if (tc::global_timer_ns() - t0 > tc::kWaitLimitNs) {
          record_status(status, kDevTimeout);
          ok = 0;
          break;
        }
      }
    }
    *ok_s = ok;
  }
  __syncthreads();
  return *ok_s != 0;
}

// Shared-memory layout (bytes) of the fused kernel: region A holds phase Q's W_q
// group and x rows, later phase G's lists and per-warp row sums; region B holds the
// scoring unit's sub-key rows and the warps' query halves.
struct FusedSmem {
  size_t a, b, total;
};
__host__ __device__ inline FusedSmem fused_smem(int d, int H, int dq, int n, int v, int esz) {
  const int half = dq / 2;
  const int nchunks = (n + kSChunk - 1) / kSChunk;
  const size_t q_bytes = static_cast<size_t>(kQFeat + kQTok) * d * esz;
  const size_t lists = static_cast<size_t>(2) * nchunks * kMaxK * 8;
  const size_t merged = static_cast<size_t>(2) * kMaxK * 8;
  const size_t picks = static_cast<size_t>(kMaxK) * 8;
  const size_t red = static_cast<size_t>(kSmallWarps) * v * 4;
  const size_t g_bytes = lists + merged + picks + red;
  FusedSmem m;
  m.a = ((q_bytes > g_bytes ? q_bytes : g_bytes) + 15) & ~static_cast<size_t>(15);
  const size_t rows = (static_cast<size_t>(esz) * kSChunk * (half + (esz == 2 ? 2 : 1)) + 15) &
                      ~static_cast<size_t>(15);
  m.b = rows + sizeof(float) * kSmallWarps * 2 * half;
  const size_t dec = sizeof(float) * kDecodeB * kSChunk;  // decode mode's chunk scores
  if (m.b < dec) m.b = dec;
  if (esz == 2) {  // the tensor-core tiles
    if (m.a < kMmaQuerySmem) m.a = kMmaQuerySmem;
    if (m.b < mma_score_smem(half)) m.b = mma_score_smem(half);
  }
  m.total = m.a + m.b + sizeof(int) * kMaxPairs;
  return m;
}

template <typename T, int MAXV>
__global__ void __launch_bounds__(kSmallWarps * 32, 1) forward_small_fused_kernel(FusedArgs a) {
  constexpr int VPER = Vec<T>::kPer;
  extern __shared__ __align__(16) unsigned char fs_raw[];
  __shared__ int ok_s;
  __shared__ int npairs_s;
  __shared__ int last_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = a.B, d = a.d, H = a.H, dq = a.dq, n = a.n, k = a.k, v = a.v;
  const int F = H * dq, half = dq >> 1;
  const int esz = static_cast<int>(sizeof(T));
  const FusedSmem L = fused_smem(d, H, dq, n, v, esz);
  unsigned char* regA = fs_raw;
  unsigned char* regB = fs_raw + L.a;
  int* pairs = reinterpret_cast<int*>(fs_raw + L.a + L.b);
  const int nchunks = (n + kSChunk - 1) / kSChunk;
  const int NQ = (F + kQFeat - 1) / kQFeat;
  const int NS = 2 * H * nchunks;
  const unsigned G = gridDim.x;
  const T* X = static_cast<const T*>(a.x);
  const T* W = static_cast<const T*>(a.W);
  const T* C = static_cast<const T*>(a.subkeys);
  const int ld = half + (sizeof(T) == 2 ? 2 : 1);  // padded sub-key row (elements)
  T* rows_s = reinterpret_cast<T*>(regB);
  float* qs = reinterpret_cast<float*>(
      regB + ((sizeof(T) * kSChunk * ld + 15) & ~static_cast<size_t>(15)));
  const int row_words_c = half * esz / 4;         // words of one sub-key row
  const int ld_words = ld * esz / 4;

  if (threadIdx.x == 0) npairs_s = build_pairs(k, pairs);
  // Per-token head counts of phase G, zeroed before the first barrier.
  if (blockIdx.x == 0)
    for (int t = threadIdx.x; t < B; t += blockDim.x) a.tok_done[t] = 0u;

  // Sub-keys of this CTA's first scoring unit: prefetched into L2 now (one request per
  // 128-byte line), since they do not depend on q; phase S stages them from there.
  if (static_cast<int>(blockIdx.x) < NS) {
    const int u = blockIdx.x;
    const int hs = u / nchunks, chunk = u - hs * nchunks;
    const int c0 = chunk * kSChunk;
    const int nr = min(kSChunk, n - c0);
    const char* src = reinterpret_cast<const char*>(C + (static_cast<int64_t>(hs) * n + c0) * half);
    const int lines = (nr * half * esz + 127) / 128;
    for (int i = threadIdx.x; i < lines; i += blockDim.x)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(src + 128 * i));
  }

  // ---------------- phase Q
  if (a.decode) {  // warp = W_q row, all tokens
    for (int f = static_cast<int>(blockIdx.x) * kSmallWarps + warp; f < F;
         f += static_cast<int>(G) * kSmallWarps)
      decode_query_row<T, kDecodeRowVecs>(X, W, a.mean, a.var, a.gamma, a.beta, a.eps, B, d,
                                          F, f, a.q);
  } else if (a.mma) {  // CTA = (16 features, 16 tokens) tiles
    float* red = reinterpret_cast<float*>(regA);
    const int nfg = F / kMmaFeat;
    const int ntiles = nfg * ((B + kMmaTok - 1) / kMmaTok);
    for (int tile = blockIdx.x; tile < ntiles; tile += G) {
      const int tg = tile / nfg, fg = tile - tg * nfg;
      mma_query_tile(reinterpret_cast<const uint16_t*>(X), reinterpret_cast<const uint16_t*>(W),
                     a.mean, a.var, a.gamma, a.beta, a.eps, B, d, F, fg * kMmaFeat,
                     tg * kMmaTok, red, a.q);
    }
  } else {
    T* ws = reinterpret_cast<T*>(regA);  // [kQFeat][d]
    T* xs = ws + kQFeat * d;             // [kQTok][d]
    const int row_words = d * esz / 4;
    for (int g = blockIdx.x; g < NQ; g += G) {
      const int f0 = g * kQFeat;
      const int nf = min(kQFeat, F - f0);
      __syncthreads();
      stage_rows(reinterpret_cast<const uint32_t*>(W + static_cast<int64_t>(f0) * d),
                 reinterpret_cast<uint32_t*>(ws), kQFeat, nf, row_words, row_words);
      for (int t0 = 0; t0 < B; t0 += kQTok) {
        __syncthreads();
        stage_rows(reinterpret_cast<const uint32_t*>(X + static_cast<int64_t>(t0) * d),
                   reinterpret_cast<uint32_t*>(xs), kQTok, min(kQTok, B - t0), row_words,
                   row_words);
        __syncthreads();
        const int t = t0 + warp;
        if (t >= B) continue;  // warp-uniform
        float acc[kQFeat];
#pragma unroll
        for (int j = 0; j < kQFeat; ++j) acc[j] = 0.f;
        const T* xr = xs + warp * d;
        if constexpr (sizeof(T) == 2) {
          const uint32_t* xw = reinterpret_cast<const uint32_t*>(xr);
          const uint32_t* ww = reinterpret_cast<const uint32_t*>(ws);
          const int dw = d >> 1;
          for (int c0 = 0; c0 < dw; c0 += 32 * 4) {
            uint32_t xv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = c0 + lane + 32 * u;
              xv[u] = c < dw ? xw[c] : 0u;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int c = c0 + lane + 32 * u;
              if (c < dw) {
                const float xa = bf16_lo(xv[u]), xb = bf16_hi(xv[u]);
#pragma unroll
                for (int j = 0; j < kQFeat; ++j) {
                  const uint32_t wv = ww[j * dw + c];
                  acc[j] = fmaf(xb, bf16_hi(wv), fmaf(xa, bf16_lo(wv), acc[j]));
                }
              }
            }
          }
        } else {
          for (int c0 = 0; c0 < d; c0 += 32 * 8) {
            float xv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int c = c0 + lane + 32 * u;
              xv[u] = c < d ? load_elem(xr, c) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int c = c0 + lane + 32 * u;
              if (c < d) {
#pragma unroll
                for (int j = 0; j < kQFeat; ++j)
                  acc[j] = fmaf(xv[u], load_elem(ws, j * d + c), acc[j]);
              }
            }
          }
        }
#pragma unroll
        for (int m = 16, c = kQFeat / 2; c >= 1; m >>= 1, c >>= 1) {
          const bool up = (lane & m) != 0;
#pragma unroll
          for (int i = 0; i < c; ++i) {
            const float send = up ? acc[i] : acc[i + c];
            const float keep = up ? acc[i + c] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
          }
        }
        const float sum = acc[0] + __shfl_xor_sync(0xffffffffu, acc[0], 1);
        const int j = lane >> 1;
        if ((lane & 1) == 0 && j < nf) {
          const int f = f0 + j;
          const float sc = a.gamma[f] / sqrtf(a.var[f] + a.eps);
          a.q[static_cast<int64_t>(t) * F + f] = fmaf(sum, sc, a.beta[f] - a.mean[f] * sc);
        }
      }
    }
  }
  if (!fused_grid_sync(a.barrier, G, a.status, &ok_s)) return;

  // ---------------- phase S
  if (a.decode) {  // warp = kDecodeKeys sub-keys, all tokens; warp t selects token t's list
    float* scs = reinterpret_cast<float*>(regB);  // [kDecodeB][kSChunk]
    for (int u = blockIdx.x; u < NS; u += G) {
      const int hs = u / nchunks, chunk = u - hs * nchunks;
      const int h = hs >> 1, side = hs & 1;
      const int c0 = chunk * kSChunk;
      uint4 kv[kDecodeKeys][kDecodeKeyVecs];
      decode_load_keys<T, kDecodeKeyVecs>(C, n, half, hs, c0, kv);
      __syncthreads();  // the previous unit's lists have been read from scs
      decode_score_keys<T, kDecodeKeyVecs>(a.q, B, F, dq, hs, kv, scs);
      __syncthreads();
      if (warp < B) {
        float s0;
        int i0;
        decode_chunk_list(scs, warp, c0, n, s0, i0);
        const int64_t o =
            ((((static_cast<int64_t>(warp) * H + h) * 2 + side) * nchunks + chunk) << 5) + lane;
        a.cs[o] = s0;
        a.ci[o] = i0;
      }
    }
  } else if (a.mma) {  // unit = (head-half, 64 sub-keys), its sub-keys in registers
    const uint16_t* Cu = reinterpret_cast<const uint16_t*>(C);
    for (int u = blockIdx.x; u < NS; u += G) {
      const int hs = u / nchunks, chunk = u - hs * nchunks;
      uint4 kf[kMmaMaxKB];
      mma_load_keys(Cu, n, half, hs, chunk * kSChunk, kf);
      for (int t0 = 0; t0 < B; t0 += kMmaTok)
        mma_score_tile(a.q, kf, B, H, dq, n, hs, chunk, t0, regB, a.cs, a.ci);
    }
  } else
  for (int u = blockIdx.x; u < NS; u += G) {
    const int hs = u / nchunks, chunk = u - hs * nchunks;
    const int h = hs >> 1, side = hs & 1;
    const int c0 = chunk * kSChunk;
    __syncthreads();
    stage_rows(reinterpret_cast<const uint32_t*>(C + (static_cast<int64_t>(hs) * n + c0) * half),
               reinterpret_cast<uint32_t*>(rows_s), kSChunk, min(kSChunk, n - c0),
               row_words_c, ld_words);
    __syncthreads();
    float* qw = qs + warp * 2 * half;
    const bool v0 = c0 + lane < n, v1 = c0 + 32 + lane < n;
    const T* r0 = rows_s + lane * ld;
    const T* r1 = rows_s + (lane + 32) * ld;
    for (int tb = warp * 2; tb < B; tb += kSmallWarps * 2) {
      // This warp's two tokens' query halves (written by other CTAs: read from L2), 16
      // loads in flight per lane before any is stored.
      for (int i0 = 0; i0 < 2 * half; i0 += 32 * 16) {
        float qv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = i0 + lane + 32 * u;
          const int uu = i / half, e = i - uu * half;
          const int t = tb + uu;
          qv[u] = (i < 2 * half && t < B)
                      ? __ldcg(a.q + static_cast<int64_t>(t) * F + h * dq + side * half + e)
                      : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = i0 + lane + 32 * u;
          if (i < 2 * half) qw[i] = qv[u];
        }
      }
      __syncwarp();
      for (int uu = 0; uu < 2; ++uu) {
        const int t = tb + uu;
        if (t >= B) break;
        const float* qq = qw + uu * half;
        float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
        for (int e = 0; e < half; e += 2) {
          const float2 qv = *reinterpret_cast<const float2*>(qq + e);
          float x0a, x0b, x1a, x1b;
          if constexpr (sizeof(T) == 2) {
            const uint32_t w0 = *reinterpret_cast<const uint32_t*>(r0 + e);
            const uint32_t w1 = *reinterpret_cast<const uint32_t*>(r1 + e);
            x0a = bf16_lo(w0); x0b = bf16_hi(w0);
            x1a = bf16_lo(w1); x1b = bf16_hi(w1);
          } else {
            x0a = load_elem(r0, e); x0b = load_elem(r0, e + 1);
            x1a = load_elem(r1, e); x1b = load_elem(r1, e + 1);
          }
          a0 = fmaf(qv.x, x0a, a0);
          a1 = fmaf(qv.x, x1a, a1);
          b0 = fmaf(qv.y, x0b, b0);
          b1 = fmaf(qv.y, x1b, b1);
        }
        a0 += b0;
        a1 += b1;
        float s0 = v0 ? a0 : -INFINITY, s1 = v1 ? a1 : -INFINITY;
        int i0 = v0 ? c0 + lane : kIdPad, i1 = v1 ? c0 + 32 + lane : kIdPad;
        warp_sort32(s0, i0);
        warp_sort32(s1, i1);
        warp_merge32(s0, i0, s1, i1);
        const int64_t o =
            ((((static_cast<int64_t>(t) * H + h) * 2 + side) * nchunks + chunk) << 5) + lane;
        a.cs[o] = s0;
        a.ci[o] = i0;
      }
      __syncwarp();
    }
  }
  if (!fused_grid_sync(a.barrier, 2 * G, a.status, &ok_s)) return;

  // ---------------- phase G: block = (token, head)
  const int list_len = 2 * nchunks * kMaxK;              // this head's two halves
  float* ls = reinterpret_cast<float*>(regA);            // [2][nchunks][32]
  int* li = reinterpret_cast<int*>(ls + list_len);
  float* ms = reinterpret_cast<float*>(li + list_len);   // [2][32] merged halves
  int* mi = reinterpret_cast<int*>(ms + 2 * kMaxK);
  int* prow = mi + 2 * kMaxK;                            // [k] picked slots
  float* pw = reinterpret_cast<float*>(prow + kMaxK);
  float* red = pw + kMaxK;                               // [8][v]
  const int nvec = v / VPER;
  const T* Vt = static_cast<const T*>(a.values);
  for (int u = blockIdx.x; u < B * H; u += G) {  // u = token * H + head
    __syncthreads();
    const int64_t src = static_cast<int64_t>(u) * list_len;
    for (int i0 = 0; i0 < list_len; i0 += blockDim.x * 4) {
      float sv[4];
      int iv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + threadIdx.x + q * blockDim.x;
        sv[q] = i < list_len ? __ldcg(a.cs + src + i) : 0.f;
        iv[q] = i < list_len ? __ldcg(a.ci + src + i) : 0;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = i0 + threadIdx.x + q * blockDim.x;
        if (i < list_len) {
          ls[i] = sv[q];
          li[i] = iv[q];
        }
      }
    }
    __syncthreads();
    // Each half's chunk lists merged as a tree over the 8 warps (as in
    // gather_small_kernel): at stride st the list at 2 st i + st is merged into the
    // list at 2 st i.
    for (int st = 1; st < nchunks; st <<= 1) {
      const int per_side = (nchunks + 2 * st - 1) / (2 * st);
      for (int item = warp; item < 2 * per_side; item += kSmallWarps) {
        const int side = item / per_side, i = item - side * per_side;
        const int a0 = 2 * st * i, b0 = a0 + st;
        if (b0 >= nchunks) continue;  // warp-uniform
        const int pa = ((side * nchunks + a0) << 5) + lane;
        const int pb = ((side * nchunks + b0) << 5) + lane;
        float bs = ls[pa];
        int bi = li[pa];
        const float cs = ls[pb];
        const int ci = li[pb];
        const float ks = __shfl_sync(0xffffffffu, bs, 31);
        const int ki = __shfl_sync(0xffffffffu, bi, 31);
        const float c0s = __shfl_sync(0xffffffffu, cs, 0);
        const int c0i = __shfl_sync(0xffffffffu, ci, 0);
        if (better(c0s, c0i, ks, ki)) warp_merge32(bs, bi, cs, ci);
        ls[pa] = bs;
        li[pa] = bi;
      }
      __syncthreads();
    }
    if (warp < 2) {
      ms[warp * kMaxK + lane] = ls[((warp * nchunks) << 5) + lane];
      mi[warp * kMaxK + lane] = li[((warp * nchunks) << 5) + lane];
    }
    __syncthreads();
    if (warp == 0) {
      float bs;
      int bi;
      select_candidates(ms[lane], mi[lane], ms[kMaxK + lane], mi[kMaxK + lane], pairs, npairs_s,
                        n, bs, bi);
      const float mx = __shfl_sync(0xffffffffu, bs, 0);
      const float e = lane < k ? expf(bs - mx) : 0.f;
      const float den = warp_sum(e);
      const float wt = e / den;
      if (lane < k) {
        const int64_t o = static_cast<int64_t>(u) * k + lane;
        a.idx[o] = bi;
        a.w[o] = wt;
        if (a.sc) a.sc[o] = bs;
        prow[lane] = bi;
        pw[lane] = wt;
      }
    }
    __syncthreads();
    // The head's k weighted rows, rows warp, warp + 8, ... all in flight at once.
    float acc[MAXV][VPER];
#pragma unroll
    for (int m = 0; m < MAXV; ++m)
#pragma unroll
      for (int e = 0; e < VPER; ++e) acc[m][e] = 0.f;
    {
      constexpr int kRows = kMaxK / kSmallWarps;  // 4
      uint4 raw[kRows][MAXV];
      float wr[kRows];
#pragma unroll
      for (int uu = 0; uu < kRows; ++uu) {
        const int r = warp + uu * kSmallWarps;
        bool live = r < k;
        int row = live ? prow[r] : 0;
        if (live && (row < 0 || row >= n * n)) {  // only reachable with NaN scores
          if (lane == 0) record_status(a.status, kDevBadSlot);
          live = false;
          row = 0;
        }
        wr[uu] = live ? pw[r] : 0.f;
        const T* rp = Vt + static_cast<int64_t>(row) * v;
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          const int vec = lane + 32 * m;
          raw[uu][m] = (live && vec < nvec) ? ld_stream_v4(rp + vec * VPER)
                                            : make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int uu = 0; uu < kRows; ++uu)
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          float f[VPER];
          Vec<T>::widen(raw[uu][m], f);
#pragma unroll
          for (int e = 0; e < VPER; ++e) acc[m][e] = fmaf(wr[uu], f[e], acc[m][e]);
        }
    }
    float* my = red + warp * v;
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
      const int vec = lane + 32 * m;
      if (vec < nvec) {
#pragma unroll
        for (int e = 0; e < VPER; ++e) my[vec * VPER + e] = acc[m][e];
      }
    }
    __syncthreads();
    float* prt = a.part + static_cast<int64_t>(u) * v;  // this head's row of the output
    for (int c = threadIdx.x; c < v; c += blockDim.x) {
      float sum = red[c];
#pragma unroll
      for (int ww = 1; ww < kSmallWarps; ++ww) sum += red[ww * v + c];
      prt[c] = sum;
    }
    // The token's last head to finish adds its H rows in head order into out (each
    // writer fences its row before the count, the last one fences before reading).
    const int t = u / H;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last_s = atomicAdd(a.tok_done + t, 1u) == static_cast<unsigned>(H - 1);
    __syncthreads();
    if (last_s) {
      __threadfence();
      const float* rows_t = a.part + static_cast<int64_t>(t) * H * v;
      for (int c = threadIdx.x * 4; c < v; c += blockDim.x * 4) {
        float4 sum = __ldcg(reinterpret_cast<const float4*>(rows_t + c));
        for (int hh = 1; hh < H; ++hh) {
          const float4 x = __ldcg(reinterpret_cast<const float4*>(rows_t + hh * v + c));
          sum = make_float4(sum.x + x.x, sum.y + x.y, sum.z + x.z, sum.w + x.w);
        }
        *reinterpret_cast<float4*>(a.out + static_cast<int64_t>(t) * v + c) = sum;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static size_t query_small_smem(int d, int dtype) {
  return static_cast<size_t>(kQFeat + kQTok) * d * (dtype == 0 ? 4 : 2);
}
static size_t score_small_smem(int dq, int dtype) {
  const int half = dq / 2;
  const size_t esz = dtype == 0 ? 4 : 2;
  const size_t rows = (esz * kSChunk * (half + (esz == 2 ? 2 : 1)) + 15) & ~static_cast<size_t>(15);
  return rows + sizeof(float) * kSmallWarps * 2 * half;
}
static size_t gather_small_smem(int n, int v) {
  const size_t list_words = static_cast<size_t>(2) * ((n + kSChunk - 1) / kSChunk) * kMaxK;
  const size_t scratch = std::max(static_cast<size_t>(kSmallWarps) * v, 2 * list_words);
  return sizeof(float) * (gather_part_len(v) + scratch) + kMaxPairs * 8 + kMaxK * 8 +
         sizeof(int) * kMaxPairs;
}

bool small_mma_shape(int d_model, int dq, int dtype) {
  return mma_shape(d_model, dq, dtype == 0 ? 4 : 2);
}

bool small_supported(int64_t B, int d_model, int H, int dq, int n, int k, int v, int dtype) {
  constexpr size_t kLimit = 200 * 1024;
  const int esz = dtype == 0 ? 4 : 2;
  // Staging copies whole 32-bit words of W_q rows and sub-key rows.
  if ((static_cast<int64_t>(d_model) * esz) % 4 || (static_cast<int64_t>(dq / 2) * esz) % 4)
    return false;
  if ((dq / 2) % 2) return false;  // the scoring loop takes element pairs
  return B >= 1 && B <= kSmallMaxB && k <= kMaxK && row_vecs_per_lane(v, dtype) > 0 &&
         query_small_smem(d_model, dtype) <= kLimit && score_small_smem(dq, dtype) <= kLimit &&
         gather_small_smem(n, v) <= kLimit && n >= 1 && H <= 8;  // H CTAs per cluster
}

size_t small_chunk_entries(int64_t B, int H, int n) {
  return static_cast<size_t>(B) * H * 2 * ((n + kSChunk - 1) / kSChunk) * kMaxK;
}

template <typename T, int MAXV, int MINB>
static cudaError_t launch_gather_small_t(const LayerArgs& a, const float* cs, const int* ci,
                                         float* out, int* idx, float* w, float* sc,
                                         cudaStream_t st) {
  const size_t smem = gather_small_smem(a.n, a.v);
  const void* kern = reinterpret_cast<const void*>(gather_small_kernel<T, MAXV, MINB>);
  cudaError_t e = set_max_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.B), a.H, 1);
  cfg.blockDim = dim3(kSmallWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = a.H;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gather_small_kernel<T, MAXV, MINB>, cs, ci,
                            static_cast<const T*>(a.values), a.H, a.n, a.k, a.v, out, idx, w,
                            sc, a.status);
}

// The default register budget keeps more loads in flight per CTA (c1024: 128 registers,
// 2 CTAs per SM, 71 clusters of 4 at once); when the B clusters would not all be
// resident at once with it, the launch takes the 4-CTA-per-SM build (64 registers)
// instead: one wave rather than a second,
// nearly empty one (47 vs 53 us per call at 112 tokens on the 1024^2 layer, while at 16
// and 64 tokens the default build is 6 and 4 us faster).
template <typename T, int MAXV>
static cudaError_t launch_gather_small(const LayerArgs& a, const float* cs, const int* ci,
                                       float* out, int* idx, float* w, float* sc,
                                       cudaStream_t st) {
  if constexpr (MAXV < 8) {
    // Clusters (the H CTAs of a token) of the default build resident at once, looked up
    // once per shared-memory size and head count.
    static std::mutex mu;
    static size_t seen_smem = 0;
    static int seen_h = 0, seen_clusters = 0;
    const size_t smem = gather_small_smem(a.n, a.v);
    int clusters = 0;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (seen_smem != smem || seen_h != a.H) {
        const void* kern = reinterpret_cast<const void*>(gather_small_kernel<T, MAXV, 1>);
        cudaError_t e = set_max_smem(kern, smem);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(1, a.H, 1);
        cfg.blockDim = dim3(kSmallWarps * 32, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 1;
        attr[0].val.clusterDim.y = a.H;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaOccupancyMaxActiveClusters(&seen_clusters, kern, &cfg);
        if (e != cudaSuccess) return e;
        seen_smem = smem;
        seen_h = a.H;
      }
      clusters = seen_clusters > 0 ? seen_clusters : 1;
    }
    if (a.B > clusters)
      return launch_gather_small_t<T, MAXV, 4>(a, cs, ci, out, idx, w, sc, st);
    return launch_gather_small_t<T, MAXV, 1>(a, cs, ci, out, idx, w, sc, st);
  } else {
    return launch_gather_small_t<T, MAXV, 2>(a, cs, ci, out, idx, w, sc, st);
  }
}

template <typename T, int MAXV>
static cudaError_t launch_fused_t(const LayerArgs& a, float* q, float* cs, int* ci, float* part,
                                  float* out, int* idx, float* w, float* sc, cudaStream_t st) {
  const FusedSmem m = fused_smem(a.d_model, a.H, a.dq, a.n, a.v, a.dtype == 0 ? 4 : 2);
  const void* kern = reinterpret_cast<const void*>(forward_small_fused_kernel<T, MAXV>);
  cudaError_t e = set_max_smem(kern, m.total);
  if (e != cudaSuccess) return e;
  FusedArgs fa;
  fa.x = a.x; fa.W = a.W_q; fa.mean = a.bn_mean; fa.var = a.bn_var; fa.gamma = a.bn_gamma;
  fa.beta = a.bn_beta; fa.subkeys = a.subkeys; fa.values = a.values; fa.eps = a.bn_eps;
  fa.B = static_cast<int>(a.B); fa.d = a.d_model; fa.H = a.H; fa.dq = a.dq; fa.n = a.n;
  fa.k = a.k; fa.v = a.v; fa.q = q; fa.cs = cs; fa.ci = ci; fa.part = part; fa.out = out;
  fa.tok_done = reinterpret_cast<unsigned*>(part + a.B * a.H * a.v);
  fa.decode = decode_mode(a.B, a.H, a.d_model, a.dq, a.dtype == 0 ? 4 : 2) ? 1 : 0;
  fa.mma = mma_mode(a.B, a.H, a.d_model, a.dq, a.dtype == 0 ? 4 : 2) ? 1 : 0;
  fa.idx = idx;
  fa.w = w; fa.sc = sc; fa.status = a.status;
  // The grid barriers' counter: the word after the status word (the caller zeroes both).
  fa.barrier = reinterpret_cast<unsigned*>(a.status + 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sm_count()), 1, 1);  // one CTA per SM
  cfg.blockDim = dim3(kSmallWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = m.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the barriers can end
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, forward_small_fused_kernel<T, MAXV>, fa);
}

bool small_fused_supported(int d_model, int H, int dq, int n, int v, int dtype) {
  const FusedSmem m = fused_smem(d_model, H, dq, n, v, dtype == 0 ? 4 : 2);
  return m.total <= 200 * 1024 && H <= kSmallWarps;
}

cudaError_t launch_forward_small_fused(const LayerArgs& a, float* q, float* chunk_s,
                                       int* chunk_i, float* part, float* out, int* idx, float* w,
                                       float* sc, cudaStream_t st) {
#define PKM_FUSED(T)                                                                     \
  switch (row_vecs_per_lane(a.v, a.dtype)) {                                             \
    case 1: return launch_fused_t<T, 1>(a, q, chunk_s, chunk_i, part, out, idx, w, sc, st);    \
    case 2: return launch_fused_t<T, 2>(a, q, chunk_s, chunk_i, part, out, idx, w, sc, st);    \
    case 4: return launch_fused_t<T, 4>(a, q, chunk_s, chunk_i, part, out, idx, w, sc, st);    \
    case 8: return launch_fused_t<T, 8>(a, q, chunk_s, chunk_i, part, out, idx, w, sc, st);    \
  }                                                                                      \
  return cudaErrorInvalidValue;
  if (a.dtype == 0) {
    PKM_FUSED(float)
  }
  PKM_FUSED(uint16_t)
#undef PKM_FUSED
}

template <typename T>
static cudaError_t launch_small_t(const LayerArgs& a, float* q, float* cs, int* ci, float* out,
                                  int* idx, float* w, float* sc, int* clear, cudaStream_t st) {
  const int F = a.H * a.dq;
  const int B = static_cast<int>(a.B);
  size_t smem = query_small_smem(a.d_model, a.dtype);
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(query_small_kernel<T>), smem);
  if (e != cudaSuccess) return e;
  const bool decode = decode_mode(B, a.H, a.d_model, a.dq, a.dtype == 0 ? 4 : 2);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kSmallWarps * 32, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (decode) {
    // 16-byte chunks per lane of a W_q row and of a sub-key row.
    const int esz = a.dtype == 0 ? 4 : 2;
    const int rv = (a.d_model * esz / 16 + 31) / 32, kv = ((a.dq / 2) * esz / 16 + 31) / 32;
    const unsigned gq = static_cast<unsigned>((F + kSmallWarps - 1) / kSmallWarps);
    const T* xp = static_cast<const T*>(a.x);
    const T* wp = static_cast<const T*>(a.W_q);
    cfg.gridDim = dim3(gq, 1, 1);
    cfg.dynamicSmemBytes = 0;
#define PKM_QDEC(RV)                                                                     \
  cudaLaunchKernelEx(&cfg, query_decode_kernel<T, RV>, xp, wp, a.bn_mean, a.bn_var,        \
                     a.bn_gamma, a.bn_beta, a.bn_eps, B, a.d_model, F, q, clear)
    e = rv <= 1 ? PKM_QDEC(1) : rv <= 2 ? PKM_QDEC(2) : rv <= 4 ? PKM_QDEC(4) : PKM_QDEC(8);
#undef PKM_QDEC
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((a.n + kSChunk - 1) / kSChunk, a.H * 2, 1);
    cfg.dynamicSmemBytes = 0;
    const float* qc = q;
    const T* kp = static_cast<const T*>(a.subkeys);
    e = kv <= 1 ? cudaLaunchKernelEx(&cfg, score_decode_kernel<T, 1>, qc, kp, B, a.H, a.dq, a.n,
                                     cs, ci)
                : cudaLaunchKernelEx(&cfg, score_decode_kernel<T, 2>, qc, kp, B, a.H, a.dq, a.n,
                                     cs, ci);
  } else if (mma_mode(B, a.H, a.d_model, a.dq, a.dtype == 0 ? 4 : 2)) {
    const int tiles = (B + kMmaTok - 1) / kMmaTok;
    const uint16_t* kp = static_cast<const uint16_t*>(a.subkeys);
    cfg.gridDim = dim3(F / kMmaFeat, tiles, 1);
    cfg.dynamicSmemBytes = 0;
    e = cudaLaunchKernelEx(&cfg, query_mma_kernel, static_cast<const uint16_t*>(a.x),
                           static_cast<const uint16_t*>(a.W_q), a.bn_mean, a.bn_var, a.bn_gamma,
                           a.bn_beta, a.bn_eps, B, a.d_model, F, q, clear);
    if (e != cudaSuccess) return e;
    smem = mma_score_smem(a.dq / 2);
    e = set_max_smem(reinterpret_cast<const void*>(score_mma_kernel), smem);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((a.n + kSChunk - 1) / kSChunk, a.H * 2, tiles);
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, score_mma_kernel, static_cast<const float*>(q), kp, B, a.H,
                           a.dq, a.n, cs, ci);
  } else {
    cfg.gridDim = dim3((F + kQFeat - 1) / kQFeat, (B + kQTok - 1) / kQTok, 1);
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, query_small_kernel<T>, static_cast<const T*>(a.x),
                           static_cast<const T*>(a.W_q), a.bn_mean, a.bn_var, a.bn_gamma,
                           a.bn_beta, a.bn_eps, B, a.d_model, F, q, clear);
    if (e != cudaSuccess) return e;
    smem = score_small_smem(a.dq, a.dtype);
    e = set_max_smem(reinterpret_cast<const void*>(score_small_kernel<T>), smem);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3((a.n + kSChunk - 1) / kSChunk, a.H * 2, (B + kSTok - 1) / kSTok);
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, score_small_kernel<T>, static_cast<const float*>(q),
                           static_cast<const T*>(a.subkeys), B, a.H, a.dq, a.n, cs, ci);
  }
  if (e != cudaSuccess) return e;
  switch (row_vecs_per_lane(a.v, a.dtype)) {
    case 1: return launch_gather_small<T, 1>(a, cs, ci, out, idx, w, sc, st);
    case 2: return launch_gather_small<T, 2>(a, cs, ci, out, idx, w, sc, st);
    case 4: return launch_gather_small<T, 4>(a, cs, ci, out, idx, w, sc, st);
    case 8: return launch_gather_small<T, 8>(a, cs, ci, out, idx, w, sc, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_forward_small(const LayerArgs& a, float* q, float* chunk_s, int* chunk_i,
                                 float* out, int* idx, float* w, float* sc, int* clear,
                                 cudaStream_t st) {
  if (a.dtype == 0)
    return launch_small_t<float>(a, q, chunk_s, chunk_i, out, idx, w, sc, clear, st);
  return launch_small_t<uint16_t>(a, q, chunk_s, chunk_i, out, idx, w, sc, clear, st);
}

}  // namespace pkm
