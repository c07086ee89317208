// pkm_gemm_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) GEMMs of the layer's backward
// through the query network ("Large Memory Layers with Product Keys", Methodology:
// the query network is a linear map trained with the rest of the model):
//
//   grad_x [B][d]  = dL/dacc [B][F] . W_q [F][d]      (M = B, N = d, K = F)
//   grad_W [F][d]  = dL/dacc^T [F][B] . x [B][d]      (M = F, N = d, K = B)
//
// dL/dacc is an fp32 result; it arrives as two bf16 planes hi + lo whose sum is within
// 2^-18 relative of it, and both planes are multiplied into one fp32 TMEM accumulator
// (x and W_q are bf16 and exact). No operand is transposed in memory: W_q and x are
// read MN-major (N = d contiguous), and dL/dacc K-major for grad_x, MN-major for
// grad_W; the MMA instruction descriptor carries the majorness.
//
// Persistent, warp-specialised, 320 threads (the layout of the query kernel):
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..9  epilogue: two warps per TMEM lane quadrant, 128 columns each
// Tiles of 128 x 256 outputs, K in blocks of 64, three 64 KiB stages, the
// accumulator double-buffered in TMEM. When the output has too few tiles to fill
// the SMs, K is split in two and both halves are added onto a zeroed output with
// float4 atomics: 0 + a + b is the same in either order, so the result stays
// deterministic. Every barrier wait is bounded as in the query kernel.
#include <mutex>

#include "pkm_common.cuh"
#include "pkm_tc.h"
#include "pkm_tcgen05.cuh"

namespace pkm {

using namespace tc;

namespace {

constexpr int kGEpiWarps = 8;
constexpr int kGThreads = 64 + 32 * kGEpiWarps;
constexpr int kGM = 128;   // MMA M
constexpr int kGN = 256;   // MMA N
constexpr int kGK = 64;    // K per stage: one 128-byte swizzled row of bf16
constexpr int kGPlanes = 2;
constexpr int kGStages = 3;
constexpr uint32_t kGAPlaneBytes = kGM * kGK * 2;             // 16 KiB
constexpr uint32_t kGABytes = kGPlanes * kGAPlaneBytes;       // 32 KiB
constexpr uint32_t kGBBytes = kGN * kGK * 2;                  // 32 KiB
constexpr uint32_t kGStageBytes = kGABytes + kGBBytes;        // 64 KiB
constexpr uint32_t kGMnBlock = 64 * kGK * 2;                  // 64 MN x 64 K: 8 KiB
constexpr uint32_t kGTmemCols = 512;

size_t gemm_tc_smem_bytes() { return 1024 + kGStages * kGStageBytes + 256; }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle: each
// 128-byte row holds 64 consecutive MN elements of one K index, 8 K rows make a
// 1024-byte swizzle atom (SBO), and successive 64-element MN blocks lie `lbo` bytes
// apart (LBO).
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t addr, uint32_t lbo) {
  const uint64_t start = (addr >> 4) & 0x3fffull;
  return start | (static_cast<uint64_t>(lbo >> 4) << 16) | ((1024ull >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

constexpr uint32_t kTransA = 1u << 15;  // A is MN-major
constexpr uint32_t kTransB = 1u << 16;  // B is MN-major

// C[M][N] (+)= sum_p A_p B^T over K. A_p: plane p of the [2][rows][F] dL/dacc planes
// (K-major when !A_MN: M = rows, K = F; MN-major when A_MN: M = F, K = rows). B: a
// [K][N] bf16 matrix read MN-major. ksplit 1 stores, 2 adds atomically.
template <bool A_MN>
__global__ void __launch_bounds__(kGThreads, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    float* __restrict__ C, int M, int N, int K, int ksplit, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kGStages * kGStageBytes);
  uint64_t* empty = full + kGStages;
  uint64_t* tfull = empty + kGStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (M + kGM - 1) / kGM;
  const int nt = (N + kGN - 1) / kGN;
  const int ntiles = mt * nt * ksplit;
  const int kblocks = (K + kGK - 1) / kGK;
  const int kper = (kblocks + ksplit - 1) / ksplit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kGEpiWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      uint32_t s = 0, ph = 0;
      uint32_t issued_phase[kGStages];
      bool issued[kGStages];
      for (int i = 0; i < kGStages; ++i) issued[i] = false;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int sp = t % ksplit, mn = t / ksplit;
        const int m0 = (mn / nt) * kGM, n0 = (mn % nt) * kGN;
        const int kb0 = sp * kper, kb1 = min(kblocks, kb0 + kper);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, status, abort)) { ok = false; break; }
          uint8_t* a = stages + s * kGStageBytes;
          uint8_t* b = a + kGABytes;
          const int k0 = kb * kGK;
          mbar_arrive_expect_tx(&full[s], kGStageBytes);
#pragma unroll
          for (int p = 0; p < kGPlanes; ++p) {
            if (A_MN) {
              tma_load_3d(a + p * kGAPlaneBytes, &tm_a, &full[s], m0, k0, p);
              tma_load_3d(a + p * kGAPlaneBytes + kGMnBlock, &tm_a, &full[s], m0 + 64, k0, p);
            } else {
              tma_load_3d(a + p * kGAPlaneBytes, &tm_a, &full[s], k0, m0, p);
            }
          }
#pragma unroll
          for (int blk = 0; blk < kGN / 64; ++blk)
            tma_load_2d(b + blk * kGMnBlock, &tm_b, &full[s], n0 + 64 * blk, k0);
          issued[s] = true;
          issued_phase[s] = ph;
          if (++s == kGStages) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int i = 0; i < kGStages; ++i)
          if (issued[i]) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[i], issued_phase[i]) &&
                   global_timer_ns() - t0 < kDrainLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kGM, kGN) | kTransB | (A_MN ? kTransA : 0u);
      uint32_t s = 0, ph = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        const int sp = t % ksplit;
        const int kb0 = sp * kper, kb1 = min(kblocks, kb0 + kper);
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[buf], tph ^ 1, status, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kGN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[s], ph, status, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_addr(stages + s * kGStageBytes);
          const uint32_t b = a + kGABytes;
#pragma unroll
          for (int j = 0; j < kGK / 16; ++j) {
            // 16 K rows = two 8-row atoms of an MN-major tile, 32 bytes of a K-major row.
            const uint64_t bd = sw128_mn_desc(b + j * 2048, kGMnBlock);
#pragma unroll
            for (int p = 0; p < kGPlanes; ++p) {
              const uint32_t ap = a + p * kGAPlaneBytes;
              const uint64_t ad = A_MN ? sw128_mn_desc(ap + j * 2048, kGMnBlock)
                                       : sw128_desc(ap, j * 32);
              mma_bf16(d_tmem, ad, bd, idesc, (kb != kb0 || j != 0 || p != 0) ? 1u : 0u);
            }
          }
          mma_commit(&empty[s]);
          if (++s == kGStages) { s = 0; ph ^= 1; }
        }
        if (ok) mma_commit(&tfull[buf]);
      }
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kDrainLimitNs) {
      }
    }
  } else {
    // ---------------- epilogue: one thread per output row, 128 columns per warp
    const int quad = warp & 3;
    const int cset = (warp - 2) >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!warp_wait(&tfull[buf], tph, status, abort)) break;
      tc_fence_after();
      const int mn = t / ksplit;
      const int m0 = (mn / nt) * kGM, n0 = (mn % nt) * kGN;
      const int row = m0 + quad * 32 + lane;
#pragma unroll 1
      for (int gg = 0; gg < 4; ++gg) {
        const int g = cset * 4 + gg;
        float v[32];
        tmem_ld32(tmem_base + lane_addr + buf * kGN + g * 32, v);
        if (gg == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        const int col = n0 + g * 32;
        if (row < M && col < N) {  // N is a multiple of 64: a 32-column group is all in or out
          float4* dst = reinterpret_cast<float4*>(C + static_cast<int64_t>(row) * N + col);
          if (ksplit == 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              atomicAdd(dst + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kGTmemCols);
  }
}

template <bool A_MN>
cudaError_t launch_gemm(const CUtensorMap& tm_a, const CUtensorMap& tm_b, float* C, int M, int N,
                        int K, int* status, cudaStream_t st) {
  const int tiles = ((M + kGM - 1) / kGM) * ((N + kGN - 1) / kGN);
  const int kblocks = (K + kGK - 1) / kGK;
  const int sms = sm_count();
  // Split K in two when one tile per SM would leave more than half of them idle.
  const int ksplit = (2 * tiles <= sms && kblocks >= 2) ? 2 : 1;
  if (ksplit == 2) {
    cudaError_t e = cudaMemsetAsync(C, 0, sizeof(float) * static_cast<size_t>(M) * N, st);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = gemm_tc_smem_bytes();
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(gemm_tc_kernel<A_MN>), smem);
  if (e != cudaSuccess) return e;
  const int units = tiles * ksplit;
  const int grid = units < sms ? units : sms;
  gemm_tc_kernel<A_MN><<<grid, kGThreads, smem, st>>>(tm_a, tm_b, C, M, N, K, ksplit, status);
  return cudaGetLastError();
}

}  // namespace

bool gemm_tc_supported(int64_t B, int F, int d) {
  return B > 0 && B < (1LL << 31) && F % kGM == 0 && d % 64 == 0 && F % kGK == 0;
}

cudaError_t launch_grad_x_tc(const void* g_planes, const void* W_q, float* grad_x, int64_t B,
                             int F, int d, int* status, cudaStream_t st) {
  CUtensorMap tm_a, tm_b;
  const cuuint64_t ad[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(B), kGPlanes};
  const cuuint64_t as[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(F) * 2 * B};
  const cuuint32_t ab[3] = {kGK, kGM, 1};                   // K-major: 64 features x 128 tokens
  const cuuint64_t bd[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(F)};
  const cuuint64_t bs[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t bb[2] = {64, kGK};                       // MN-major: 64 columns x 64 K rows
  if (!make_map(&tm_a, g_planes, 3, ad, as, ab) || !make_map(&tm_b, W_q, 2, bd, bs, bb))
    return cudaErrorInvalidValue;
  return launch_gemm<false>(tm_a, tm_b, grad_x, static_cast<int>(B), d, F, status, st);
}

cudaError_t launch_grad_w_tc(const void* g_planes, const void* x, float* grad_W, int64_t B,
                             int F, int d, int* status, cudaStream_t st) {
  CUtensorMap tm_a, tm_b;
  const cuuint64_t ad[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(B), kGPlanes};
  const cuuint64_t as[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(F) * 2 * B};
  const cuuint32_t ab[3] = {64, kGK, 1};                    // MN-major: 64 features x 64 tokens
  const cuuint64_t bd[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(B)};
  const cuuint64_t bs[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t bb[2] = {64, kGK};
  if (!make_map(&tm_a, g_planes, 3, ad, as, ab) || !make_map(&tm_b, x, 2, bd, bs, bb))
    return cudaErrorInvalidValue;
  return launch_gemm<true>(tm_a, tm_b, grad_W, F, d, static_cast<int>(B), status, st);
}

}  // namespace pkm
