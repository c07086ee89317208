// pkm_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) kernels for sm_100a:
//
//   query_tc_kernel        q = BN(x W_q^T), written as three bf16 planes hi/mid/lo
//   score_topk_tc_kernel   s = q_half C^T per (128-token tile, head, half), scored in
//                          256-sub-key chunks into TMEM, with the per-row top-k kept
//                          in registers: the scores never reach HBM
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology and the
// Deep Analysis / Methodology list): the query network q(x) is a linear map with
// BatchNorm ("batch normalization in the query network"); q is split into q1, q2;
// each half runs an inner-product search against its own sub-key set and keeps its
// top-k sub-keys.
//
// Both kernels are persistent (one CTA per SM) and warp-specialised, 192 threads:
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..5  epilogue, one thread per accumulator row (TMEM lane)
// Operands are staged by TMA with the 128-byte swizzle; the accumulator is double
// buffered in TMEM (2 x 256 fp32 columns) so the epilogue of one tile overlaps the
// MMAs of the next. Every barrier wait is bounded (pkm_tcgen05.cuh); on a timeout
// the kernel records it in the status word, stops issuing work, waits (bounded) for
// its own copies and MMAs in flight, frees TMEM and exits.
//
// Precision: q is an fp32 result. Rounding it to bf16 before scoring would move
// scores by ~1e-3 relative, far more than the gaps that decide which keys are
// kept, so the query kernel writes q = hi + mid + lo (three bf16 values, exact to
// ~2^-24 relative) and the scoring kernel issues three MMAs per K step into one fp32
// accumulator. Sub-keys are bf16 and exact.
#include <mutex>

#include "pkm_common.cuh"
#include "pkm_tc.h"
#include "pkm_tcgen05.cuh"

namespace pkm {

using namespace tc;

constexpr int kTcThreads = 192;
constexpr int kRowsPerTile = 128;  // MMA M (one TMEM lane per row)
constexpr int kColsPerMma = 256;   // MMA N
constexpr int kKBlock = 64;        // bf16 elements per 128-byte swizzled row
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ===========================================================================
// Query network: q = BN(x W_q^T) -> bf16 planes [3][B][F]
// ===========================================================================
constexpr int kQStages = 4;
constexpr uint32_t kQABytes = kRowsPerTile * kKBlock * 2;  // 16 KiB
constexpr uint32_t kQBBytes = kColsPerMma * kKBlock * 2;   // 32 KiB
constexpr uint32_t kQStageBytes = kQABytes + kQBBytes;
constexpr int kQMaxF = 4096;  // BN scale/shift of every feature live in shared memory

size_t query_tc_smem_bytes() {
  return 1024 + kQStages * kQStageBytes + 2 * kQMaxF * sizeof(float) + 256;
}

__global__ void __launch_bounds__(kTcThreads, 1) query_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
    const float* __restrict__ mean, const float* __restrict__ var,
    const float* __restrict__ gamma, const float* __restrict__ beta, float eps, int B, int d,
    int F, uint16_t* __restrict__ planes, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = align1024(smem_raw);
  float* scale_s = reinterpret_cast<float*>(stages + kQStages * kQStageBytes);
  float* shift_s = scale_s + kQMaxF;
  uint64_t* full = reinterpret_cast<uint64_t*>(shift_s + kQMaxF);
  uint64_t* empty = full + kQStages;
  uint64_t* tfull = empty + kQStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (B + kRowsPerTile - 1) / kRowsPerTile;
  const int nt = F / kColsPerMma;
  const int ntiles = mt * nt;
  const int kiters = d / kKBlock;

  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float sc = gamma[f] / sqrtf(var[f] + eps);
    scale_s[f] = sc;
    shift_s[f] = beta[f] - mean[f] * sc;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
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
      uint32_t issued_phase[kQStages];
      bool issued[kQStages];
      for (int i = 0; i < kQStages; ++i) issued[i] = false;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int m = t / nt, nn = t - m * nt;
        for (int kb = 0; kb < kiters; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, status, abort)) { ok = false; break; }
          uint8_t* a = stages + s * kQStageBytes;
          mbar_arrive_expect_tx(&full[s], kQStageBytes);
          tma_load_2d(a, &tm_x, &full[s], kb * kKBlock, m * kRowsPerTile);
          tma_load_2d(a + kQABytes, &tm_w, &full[s], kb * kKBlock, nn * kColsPerMma);
          issued[s] = true;
          issued_phase[s] = ph;
          if (++s == kQStages) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int i = 0; i < kQStages; ++i)
          if (issued[i]) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[i], issued_phase[i]) &&
                   global_timer_ns() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kRowsPerTile, kColsPerMma);
      uint32_t s = 0, ph = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[buf], tph ^ 1, status, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kColsPerMma;
        for (int kb = 0; kb < kiters; ++kb) {
          if (!mbar_wait(&full[s], ph, status, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = smem_addr(stages + s * kQStageBytes);
          const uint32_t b = a + kQABytes;
#pragma unroll
          for (int j = 0; j < kKBlock / 16; ++j)
            mma_bf16(d_tmem, sw128_desc(a, j * 32), sw128_desc(b, j * 32), idesc,
                     (kb | j) != 0);
          mma_commit(&empty[s]);
          if (++s == kQStages) { s = 0; ph ^= 1; }
        }
        if (ok) mma_commit(&tfull[buf]);
      }
      // Wait (bounded) until every MMA issued above has finished reading shared memory
      // and writing TMEM before the CTA tears down.
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // ---------------- epilogue: BN affine + 3-plane split, one thread per row
    const int quad = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const size_t plane_stride = static_cast<size_t>(B) * F;
    int it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!warp_wait(&tfull[buf], tph, status, abort)) break;
      tc_fence_after();
      const int m = t / nt, nn = t - m * nt;
      const int64_t row = static_cast<int64_t>(m) * kRowsPerTile + quad * 32 + lane;
#pragma unroll 1
      for (int g = 0; g < kColsPerMma / 32; ++g) {
        float v[32];
        tmem_ld32(tmem_base + lane_addr + buf * kColsPerMma + g * 32, v);
        if (g == kColsPerMma / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        if (row < B) {
          const int f0 = nn * kColsPerMma + g * 32;
          uint32_t ph_[16], pm[16], pl[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float q0 = fmaf(v[i], scale_s[f0 + i], shift_s[f0 + i]);
            const float q1 = fmaf(v[i + 1], scale_s[f0 + i + 1], shift_s[f0 + i + 1]);
            uint16_t h0, m0, l0, h1, m1, l1;
            split3(q0, h0, m0, l0);
            split3(q1, h1, m1, l1);
            ph_[i / 2] = h0 | (static_cast<uint32_t>(h1) << 16);
            pm[i / 2] = m0 | (static_cast<uint32_t>(m1) << 16);
            pl[i / 2] = l0 | (static_cast<uint32_t>(l1) << 16);
          }
          uint16_t* dst = planes + row * F + f0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            reinterpret_cast<uint4*>(dst)[c] =
                make_uint4(ph_[4 * c], ph_[4 * c + 1], ph_[4 * c + 2], ph_[4 * c + 3]);
            reinterpret_cast<uint4*>(dst + plane_stride)[c] =
                make_uint4(pm[4 * c], pm[4 * c + 1], pm[4 * c + 2], pm[4 * c + 3]);
            reinterpret_cast<uint4*>(dst + 2 * plane_stride)[c] =
                make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
          }
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ===========================================================================
// Per-half scores and top-k
// ===========================================================================
constexpr int kSStages = 2;
constexpr uint32_t kSPlaneBytes = kRowsPerTile * kKBlock * 2;      // 16 KiB
constexpr uint32_t kSABytes = 3 * kSPlaneBytes;                     // 48 KiB
constexpr uint32_t kSBBytes = kColsPerMma * kKBlock * 2;            // 32 KiB
constexpr uint32_t kSStageBytes = kSABytes + kSBBytes;              // 80 KiB
constexpr int kSCap = 64;  // survivors buffered per row before they are merged

size_t score_tc_smem_bytes() {
  return 1024 + kSStages * kSStageBytes + 2 * kSCap * kRowsPerTile * sizeof(float) + 256;
}

// Sort 32 (score, id) pairs held by one thread, best first (bitonic network).
__device__ __forceinline__ void thread_sort32(float (&s)[32], int (&id)[32]) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0 || size == 32;
          const bool jb = better(s[j], id[j], s[i], id[i]);
          const bool sw = desc ? jb : better(s[i], id[i], s[j], id[j]);
          const float ts = sw ? s[j] : s[i];
          const int ti = sw ? id[j] : id[i];
          s[j] = sw ? s[i] : s[j];
          id[j] = sw ? id[i] : id[j];
          s[i] = ts;
          id[i] = ti;
        }
      }
}

// Keep the best 32 of the sorted list L and the sorted batch b; L stays sorted.
__device__ __forceinline__ void thread_merge32(float (&Ls)[32], int (&Li)[32],
                                               const float (&bs)[32], const int (&bi)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const bool take = better(bs[31 - i], bi[31 - i], Ls[i], Li[i]);
    Ls[i] = take ? bs[31 - i] : Ls[i];
    Li[i] = take ? bi[31 - i] : Li[i];
  }
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1)
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int j = i ^ stride;
      if (j > i) {
        const bool sw = better(Ls[j], Li[j], Ls[i], Li[i]);
        const float ts = sw ? Ls[j] : Ls[i];
        const int ti = sw ? Li[j] : Li[i];
        Ls[j] = sw ? Ls[i] : Ls[j];
        Li[j] = sw ? Li[i] : Li[j];
        Ls[i] = ts;
        Li[i] = ti;
      }
    }
}

// Merge this thread's buffered survivors (cnt of them) into L, 32 at a time. Called by
// all lanes of the warp together.
__device__ __forceinline__ void absorb_survivors(float (&Ls)[32], int (&Li)[32],
                                                 const float* sv_s, const int* sv_i, int cnt,
                                                 int r) {
#pragma unroll 1
  for (int b0 = 0; b0 < kSCap; b0 += 32) {
    if (!__any_sync(0xffffffffu, cnt > b0)) break;
    float bs[32];
    int bi[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool ok = b0 + j < cnt;
      bs[j] = ok ? sv_s[(b0 + j) * kRowsPerTile + r] : -INFINITY;
      bi[j] = ok ? sv_i[(b0 + j) * kRowsPerTile + r] : kIdPad;
    }
    thread_sort32(bs, bi);
    thread_merge32(Ls, Li, bs, bi);
  }
}

__global__ void __launch_bounds__(kTcThreads, 1) score_topk_tc_kernel(
    const __grid_constant__ CUtensorMap tm_planes, const __grid_constant__ CUtensorMap tm_keys,
    int B, int H, int dq, int n, int k, float* __restrict__ list_s, int* __restrict__ list_i,
    int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = align1024(smem_raw);
  float* sv_s = reinterpret_cast<float*>(stages + kSStages * kSStageBytes);  // [kSCap][128]
  int* sv_i = reinterpret_cast<int*>(sv_s + kSCap * kRowsPerTile);           // [kSCap][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(sv_i + kSCap * kRowsPerTile);
  uint64_t* empty = full + kSStages;
  uint64_t* tfull = empty + kSStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = dq / 2;
  const int mt = (B + kRowsPerTile - 1) / kRowsPerTile;
  const int HS = 2 * H;
  const int nunits = mt * HS;
  const int nchunks = n / kColsPerMma;
  const int kiters = half / kKBlock;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_planes);
    prefetch_tensormap(&tm_keys);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: per K step three q planes + one sub-key tile
      uint32_t s = 0, ph = 0;
      uint32_t issued_phase[kSStages];
      bool issued[kSStages];
      for (int i = 0; i < kSStages; ++i) issued[i] = false;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const int m = u / HS, hs = u - m * HS;
        const int h = hs >> 1, side = hs & 1;
        const int xq = h * dq + side * half;
        for (int c = 0; c < nchunks && ok; ++c)
          for (int kb = 0; kb < kiters; ++kb) {
            if (!mbar_wait(&empty[s], ph ^ 1, status, abort)) { ok = false; break; }
            uint8_t* a = stages + s * kSStageBytes;
            mbar_arrive_expect_tx(&full[s], kSStageBytes);
#pragma unroll
            for (int p = 0; p < 3; ++p)
              tma_load_3d(a + p * kSPlaneBytes, &tm_planes, &full[s], xq + kb * kKBlock,
                          m * kRowsPerTile, p);
            tma_load_2d(a + kSABytes, &tm_keys, &full[s], kb * kKBlock, hs * n + c * kColsPerMma);
            issued[s] = true;
            issued_phase[s] = ph;
            if (++s == kSStages) { s = 0; ph ^= 1; }
          }
      }
      if (!ok) {
        for (int i = 0; i < kSStages; ++i)
          if (issued[i]) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[i], issued_phase[i]) &&
                   global_timer_ns() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: chunk of 256 sub-keys = kiters x 3 planes x 4 MMAs
      const uint32_t idesc = idesc_bf16_f32(kRowsPerTile, kColsPerMma);
      uint32_t s = 0, ph = 0;
      bool ok = true;
      int ci = 0;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x)
        for (int c = 0; c < nchunks && ok; ++c, ++ci) {
          const int buf = ci & 1;
          const uint32_t tph = (ci >> 1) & 1;
          if (!mbar_wait(&tempty[buf], tph ^ 1, status, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + buf * kColsPerMma;
          for (int kb = 0; kb < kiters; ++kb) {
            if (!mbar_wait(&full[s], ph, status, abort)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a = smem_addr(stages + s * kSStageBytes);
            const uint32_t b = a + kSABytes;
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
              for (int j = 0; j < kKBlock / 16; ++j)
                mma_bf16(d_tmem, sw128_desc(a + p * kSPlaneBytes, j * 32),
                         sw128_desc(b, j * 32), idesc, (kb | p | j) != 0);
            mma_commit(&empty[s]);
            if (++s == kSStages) { s = 0; ph ^= 1; }
          }
          if (ok) mma_commit(&tfull[buf]);
        }
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // ---------------- epilogue: running top-k per row (= TMEM lane)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    int ci = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
      const int m = u / HS, hs = u - m * HS;
      float Ls[32];
      int Li[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) { Ls[i] = -INFINITY; Li[i] = kIdPad; }
      float tau = -INFINITY;  // score of the current 32nd best: anything not above it loses
      int cnt = 0;
      for (int c = 0; c < nchunks; ++c, ++ci) {
        const int buf = ci & 1;
        const uint32_t tph = (ci >> 1) & 1;
        if (!warp_wait(&tfull[buf], tph, status, abort)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int g = 0; g < kColsPerMma / 32; ++g) {
          float v[32];
          tmem_ld32(tmem_base + lane_addr + buf * kColsPerMma + g * 32, v);
          if (g == kColsPerMma / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
          }
          // Columns arrive in increasing sub-key id, so a score equal to tau has a larger
          // id than the 32nd best and loses: strict comparison is exact.
          const int id0 = c * kColsPerMma + g * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (v[i] > tau) {
              sv_s[cnt * kRowsPerTile + r] = v[i];
              sv_i[cnt * kRowsPerTile + r] = id0 + i;
              ++cnt;
            }
          }
          if (__any_sync(0xffffffffu, cnt >= 32)) {
            absorb_survivors(Ls, Li, sv_s, sv_i, cnt, r);
            cnt = 0;
            tau = Ls[31];
          }
        }
      }
      if (!ok) break;
      absorb_survivors(Ls, Li, sv_s, sv_i, cnt, r);
      const int64_t row = static_cast<int64_t>(m) * kRowsPerTile + r;
      if (row < B) {
        const int64_t o = (row * HS + hs) * static_cast<int64_t>(k);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < k) {
            list_s[o + j] = Ls[j];
            list_i[o + j] = Li[j];
          }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ===========================================================================
// Host side: tensor maps and launches
// ===========================================================================
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor map with a {64 x rows} box and the 128-byte swizzle. dims/strides are
// innermost first; strides are in bytes for dims 1.. (dim 0 is contiguous).
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static std::once_flag once;
  static int n = 148;
  std::call_once(once, [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      n = v;
  });
  return n;
}

}  // namespace

bool tc_supported(int dtype, int d_model, int H, int dq, int n, int k) {
  if (dtype != 1) return false;
  if (d_model % kKBlock || (dq / 2) % kKBlock || n % kColsPerMma || k > 32) return false;
  const int64_t F = static_cast<int64_t>(H) * dq;
  if (F % kColsPerMma || F > kQMaxF) return false;
  if (static_cast<int64_t>(H) * 2 * n > (1LL << 31) - 1) return false;
  return true;
}

cudaError_t launch_query_tc(const LayerArgs& a, void* planes, cudaStream_t st) {
  const int F = a.H * a.dq;
  CUtensorMap tm_x, tm_w;
  const cuuint64_t xd[2] = {static_cast<cuuint64_t>(a.d_model), static_cast<cuuint64_t>(a.B)};
  const cuuint64_t xs[1] = {static_cast<cuuint64_t>(a.d_model) * 2};
  const cuuint32_t xb[2] = {kKBlock, kRowsPerTile};
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(a.d_model), static_cast<cuuint64_t>(F)};
  const cuuint32_t wb[2] = {kKBlock, kColsPerMma};
  if (!make_map(&tm_x, a.x, 2, xd, xs, xb) || !make_map(&tm_w, a.W_q, 2, wd, xs, wb))
    return cudaErrorInvalidValue;
  const size_t smem = query_tc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(query_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((a.B + kRowsPerTile - 1) / kRowsPerTile) * (F / kColsPerMma);
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  query_tc_kernel<<<grid, kTcThreads, smem, st>>>(tm_x, tm_w, a.bn_mean, a.bn_var, a.bn_gamma,
                                                  a.bn_beta, a.bn_eps, static_cast<int>(a.B),
                                                  a.d_model, F, static_cast<uint16_t*>(planes),
                                                  a.status);
  return cudaGetLastError();
}

cudaError_t launch_score_topk_tc(const LayerArgs& a, const void* planes, float* list_s,
                                 int* list_i, cudaStream_t st) {
  const int F = a.H * a.dq;
  const int half = a.dq / 2;
  CUtensorMap tm_p, tm_k;
  const cuuint64_t pd[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(a.B), 3};
  const cuuint64_t ps[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(F) * 2 * a.B};
  const cuuint32_t pb[3] = {kKBlock, kRowsPerTile, 1};
  const cuuint64_t kd[2] = {static_cast<cuuint64_t>(half),
                            static_cast<cuuint64_t>(a.H) * 2 * a.n};
  const cuuint64_t ks[1] = {static_cast<cuuint64_t>(half) * 2};
  const cuuint32_t kbx[2] = {kKBlock, kColsPerMma};
  if (!make_map(&tm_p, planes, 3, pd, ps, pb) || !make_map(&tm_k, a.subkeys, 2, kd, ks, kbx))
    return cudaErrorInvalidValue;
  const size_t smem = score_tc_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(score_topk_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = ((a.B + kRowsPerTile - 1) / kRowsPerTile) * 2 * a.H;
  const int grid = static_cast<int>(units < sm_count() ? units : sm_count());
  score_topk_tc_kernel<<<grid, kTcThreads, smem, st>>>(tm_p, tm_k, static_cast<int>(a.B), a.H,
                                                       a.dq, a.n, a.k, list_s, list_i, a.status);
  return cudaGetLastError();
}

}  // namespace pkm
