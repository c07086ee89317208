// pkm_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) kernels for sm_100a:
//
//   query_tc_kernel        q = BN(x W_q^T), written as bf16 planes hi/lo (the forward)
//                          or acc = x W_q^T as hi/mid/lo (batch statistics, backward)
//   score_topk_tc_kernel   s = q_half C^T per (128-token tile, head, half), scored in
//                          256-sub-key chunks into TMEM; one epilogue thread per row
//                          keeps the row's best 32 sub-keys: the scores never reach HBM
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology and the
// Deep Analysis / Methodology list): the query network q(x) is a linear map with
// BatchNorm ("batch normalization in the query network"); q is split into q1, q2;
// each half runs an inner-product search against its own sub-key set and keeps its
// top-k sub-keys.
//
// Both kernels are persistent (one CTA per SM) and warp-specialised, 320 threads:
//   warp 0      TMA producer (one elected lane)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..9  epilogue: two warps per TMEM lane quadrant, one thread per
//               accumulator row; each of the two takes half of every chunk's columns
// Operands are staged by TMA with the 128-byte swizzle; the accumulator is double
// buffered in TMEM (2 x 256 fp32 columns) so the epilogue of one tile overlaps the
// MMAs of the next. Every barrier wait is bounded (pkm_tcgen05.cuh); on a timeout
// the kernel records it in the status word, stops issuing work, waits (bounded) for
// its own copies and MMAs in flight, frees TMEM and exits.
//
// Precision: q is an fp32 result. Rounding it to bf16 before scoring would move
// scores by ~1e-3 relative, far more than the gaps that decide which keys are
// kept, so the query kernel writes q = hi + lo (hi = RN(q), lo = RN(q - hi): the
// residual is at most 2^-16 |q|, about 2^-18 |q| on average) and the scoring kernel
// issues two MMAs per K step into one fp32 accumulator. That residual is at the
// level of the tensor cores' own fp32 accumulation error on these sums (about
// 1e-5 absolute on per-half scores near 3), and far below the 1e-5 relative window
// in which two keys count as tied. Sub-keys are bf16 and exact.
#include <mutex>

#include "pkm_common.cuh"
#include "pkm_tc.h"
#include "pkm_tcgen05.cuh"

namespace pkm {

using namespace tc;

constexpr int kEpiWarps = 8;
constexpr int kTcThreads = 64 + 32 * kEpiWarps;
constexpr int kRowsPerTile = 128;  // MMA M (one TMEM lane per row)
constexpr int kColsPerMma = 256;   // MMA N
constexpr int kKBlock = 64;        // bf16 elements per 128-byte swizzled row
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ===========================================================================
// Query network: q = BN(x W_q^T) -> NP bf16 planes [NP][B][F]
// ===========================================================================
constexpr uint32_t kQABytes = kRowsPerTile * kKBlock * 2;  // 16 KiB
constexpr uint32_t kQBBytes = kColsPerMma * kKBlock * 2;   // 32 KiB
constexpr uint32_t kQStageBytes = kQABytes + kQBBytes;
constexpr int kQMaxF = 4096;  // features (the planes' row length fits one tensor map box run)
// Output staging: per epilogue warp, its 32 rows x 32 columns of each plane (64-byte
// rows, 64-byte swizzle), written to HBM by TMA tensor stores.
constexpr uint32_t kQStagePlane = 32 * 32 * 2;             // 2 KiB
// Operand stages: four with two output planes (the forward), three with three.
__host__ __device__ constexpr int query_stages(int np) { return np == 2 ? 4 : 3; }

template <int NP>
size_t query_tc_smem_bytes() {
  return 1024 + query_stages(NP) * kQStageBytes + kEpiWarps * NP * kQStagePlane + 256;
}

// NP = 2: q = BN(acc) as hi, mid (the forward's scoring planes); NP = 3: acc itself
// (raw_acc) as hi, mid, lo. The BatchNorm scale and shift of a column are formed in the
// epilogue from the parameters in global memory (L1-resident after the first tiles),
// so shared memory holds only operand stages and output staging.
template <int NP>
__global__ void __launch_bounds__(kTcThreads, 1) query_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
    const __grid_constant__ CUtensorMap tm_out, const float* __restrict__ mean,
    const float* __restrict__ var, const float* __restrict__ gamma,
    const float* __restrict__ beta, float eps, int B, int d, int F, int raw_acc,
    int* status) {
  constexpr int kQStages = query_stages(NP);
  constexpr uint32_t kQStageWarp = NP * kQStagePlane;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = align1024(smem_raw);
  uint8_t* staging = stages + kQStages * kQStageBytes;  // [kEpiWarps][NP planes]
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kEpiWarps * kQStageWarp);
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
    prefetch_tensormap(&tm_out);
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
                   global_timer_ns() - t0 < kDrainLimitNs) {
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
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kDrainLimitNs) {
      }
    }
  } else {
    // ---------------- epilogue: BN affine + 3-plane split, one thread per row
    const int quad = warp & 3;
    const int cset = (warp - 2) >> 2;  // which half of the 256 columns this warp converts
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    constexpr int kGroups = kColsPerMma / 32 / 2;  // 32-column groups per warp
    uint8_t* stg = staging + (warp - 2) * kQStageWarp;
    // This lane's row inside the staging tile; chunk c (8 columns, 16 bytes) of it sits
    // at position c ^ ((lane >> 1) & 3): the 64-byte swizzle the store map expects.
    uint8_t* my_row = stg + lane * 64;
    const int swz = (lane >> 1) & 3;
    int it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!warp_wait(&tfull[buf], tph, status, abort)) break;
      tc_fence_after();
      const int m = t / nt, nn = t - m * nt;
#pragma unroll 1
      for (int gg = 0; gg < kGroups; ++gg) {
        const int g = cset * kGroups + gg;
        float v[32];
        tmem_ld32(tmem_base + lane_addr + buf * kColsPerMma + g * 32, v);
        if (gg == kGroups - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        const int f0 = nn * kColsPerMma + g * 32;
        uint32_t ph_[16], pm[16], pl[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          float q[4] = {v[i], v[i + 1], v[i + 2], v[i + 3]};
          if (!raw_acc) {
            const float4 gm = __ldg(reinterpret_cast<const float4*>(gamma + f0 + i));
            const float4 vr = __ldg(reinterpret_cast<const float4*>(var + f0 + i));
            const float4 mu = __ldg(reinterpret_cast<const float4*>(mean + f0 + i));
            const float4 bt = __ldg(reinterpret_cast<const float4*>(beta + f0 + i));
            const float g4[4] = {gm.x, gm.y, gm.z, gm.w}, v4[4] = {vr.x, vr.y, vr.z, vr.w};
            const float m4[4] = {mu.x, mu.y, mu.z, mu.w}, b4[4] = {bt.x, bt.y, bt.z, bt.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              // rsqrtf: a few ulp from 1/sqrt, far below the 2^-16 |q| of the planes' split.
              const float sc = g4[u] * rsqrtf(v4[u] + eps);
              q[u] = fmaf(q[u], sc, b4[u] - m4[u] * sc);
            }
          }
          // hi = RN(q), mid = RN(q - hi), lo = RN(q - hi - mid); the forward's two
          // planes are hi and mid.
          split3_pair(q[0], q[1], ph_[i / 2], pm[i / 2], pl[i / 2]);
          split3_pair(q[2], q[3], ph_[i / 2 + 1], pm[i / 2 + 1], pl[i / 2 + 1]);
        }
        // The previous group's stores must have read the staging tile before it is
        // overwritten.
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int pos = (c ^ swz) * 16;
          *reinterpret_cast<uint4*>(my_row + pos) =
              make_uint4(ph_[4 * c], ph_[4 * c + 1], ph_[4 * c + 2], ph_[4 * c + 3]);
          *reinterpret_cast<uint4*>(my_row + kQStagePlane + pos) =
              make_uint4(pm[4 * c], pm[4 * c + 1], pm[4 * c + 2], pm[4 * c + 3]);
          if (NP == 3)
            *reinterpret_cast<uint4*>(my_row + 2 * kQStagePlane + pos) =
                make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int row0 = m * kRowsPerTile + quad * 32;
        if (lane == 0 && row0 < B) {
          // Rows past B in a partly filled box lie outside the tensor map and are not
          // written; a box that starts past B is not issued at all.
#pragma unroll
          for (int p = 0; p < NP; ++p) tma_store_3d(&tm_out, stg + p * kQStagePlane, f0, row0, p);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait0();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ===========================================================================
// Per-half scores and the best 32 per row
// ===========================================================================
// Two epilogue warp sets work on alternate units of the CTA, each with its own TMEM
// accumulator (256 columns) and its own survivor log, so two warps share each SM
// sub-partition. The MMA issuer interleaves the two sets' chunks.
constexpr int kSSets = 2;
constexpr int kSEpiWarps = 4 * kSSets;
constexpr int kSThreads = 64 + 32 * kSEpiWarps;
constexpr int kSK = 32;                                             // K per stage
constexpr int kSStages = 3;
constexpr CUtensorMapSwizzle kSSwizzle = CU_TENSOR_MAP_SWIZZLE_64B;
constexpr uint32_t kSPlaneBytes = kRowsPerTile * kSK * 2;           // 8 KiB
constexpr uint32_t kSABytes = kScorePlanes * kSPlaneBytes;          // 16 KiB
constexpr uint32_t kSBBytes = kColsPerMma * kSK * 2;                // 16 KiB
constexpr uint32_t kSStageBytes = kSABytes + kSBBytes;              // 32 KiB
constexpr int kList = kMaxK;          // entries per per-half list (the best 32, any order)
constexpr int kSStep = 8;             // columns read from TMEM per step
constexpr int kSSteps = kColsPerMma / kSStep;  // steps per chunk
constexpr int kSNewCap = 48;          // survivors logged between two merges
constexpr int kSEndMerge = 8;         // fresh entries worth a merge at a chunk's end
constexpr int kSLogCap = kList + kSNewCap;
constexpr int kSMidMerge = kSNewCap - 2 * kSStep;  // fresh entries that force a merge
                                                   // inside a chunk
constexpr int kSFull = kSLogCap - 2 * kSStep;      // entries that force one (room for two
                                                   // more steps left)
constexpr int kSCompactAt = kSLogCap - 4 * kSStep; // entries above which a merge compacts
constexpr int kSTrash = kSLogCap;     // slot written (and dropped) past a full log
constexpr int kSLogRows = kSLogCap + 1;
static_assert(kSSteps % 2 == 0, "the step loop alternates two load buffers");

size_t score_tc_smem_bytes() {
  // stages + per-set log: fp32 scores and 16-bit ids for 128 rows + barriers
  return 1024 + kSStages * kSStageBytes + kSSets * kSLogRows * kRowsPerTile * (4 + 2) + 256;
}

// Sort 32 floats held by one thread, largest first (bitonic network of min/max).
__device__ __forceinline__ void thread_sort32f(float (&x)[32]) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0 || size == 32;
          const float a = x[i], b = x[j];
          x[i] = desc ? fmaxf(a, b) : fminf(a, b);
          x[j] = desc ? fminf(a, b) : fmaxf(a, b);
        }
      }
}

// Sort 16 floats held by one thread, largest first.
__device__ __forceinline__ void thread_sort16f(float (&x)[16]) {
#pragma unroll
  for (int size = 2; size <= 16; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0 || size == 16;
          const float a = x[i], b = x[j];
          x[i] = desc ? fmaxf(a, b) : fminf(a, b);
          x[j] = desc ? fminf(a, b) : fmaxf(a, b);
        }
      }
}

// 32nd largest of 64 floats: sort both halves, then the elementwise max of one half
// and the other reversed is the best 32 (as a set); its minimum is the answer.
__device__ __forceinline__ float kth32_of_64(float (&x)[64]) {
  float a[32], b[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) { a[i] = x[i]; b[i] = x[32 + i]; }
  thread_sort32f(a);
  thread_sort32f(b);
  float t = INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i) t = fminf(t, fmaxf(a[i], b[31 - i]));
  return t;
}

__global__ void __launch_bounds__(kSThreads, 1) score_topk_tc_kernel(
    const __grid_constant__ CUtensorMap tm_planes, const __grid_constant__ CUtensorMap tm_keys,
    int B, int H, int dq, int n, float* __restrict__ list_s, int* __restrict__ list_i,
    int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stages = align1024(smem_raw);
  // per set: log scores [kSLogRows][128], then (after both sets) log ids [kSLogRows][128]
  float* lg_s_all = reinterpret_cast<float*>(stages + kSStages * kSStageBytes);
  uint16_t* lg_i_all = reinterpret_cast<uint16_t*>(lg_s_all + kSSets * kSLogRows * kRowsPerTile);
  uint64_t* full = reinterpret_cast<uint64_t*>(lg_i_all + kSSets * kSLogRows * kRowsPerTile);
  uint64_t* empty = full + kSStages;
  uint64_t* tfull = empty + kSStages;   // [2] one per TMEM accumulator
  uint64_t* tempty = tfull + 2;         // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = dq / 2;
  const int mt = (B + kRowsPerTile - 1) / kRowsPerTile;
  const int HS = 2 * H;
  const int nunits = mt * HS;
  const int nchunks = n / kColsPerMma;
  const int kiters = half / kSK;
  // This CTA's units are nunits - 1 - (blockIdx.x + j * gridDim.x); set s takes the j
  // with j % 2 == s. Units run from the last token tile down: the query kernel writes
  // the q planes in tile order, so the most recently written tiles, the ones most
  // likely still in L2, are scored first.
  const int myunits = nunits > static_cast<int>(blockIdx.x)
                          ? (nunits - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1
                          : 0;

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
      // ---------------- TMA producer: per K step the q planes + one sub-key tile, in
      // the order the MMA issuer consumes them (chunks of the two sets interleaved)
      uint32_t s = 0, ph = 0;
      uint32_t issued_phase[kSStages];
      bool issued[kSStages];
      for (int i = 0; i < kSStages; ++i) issued[i] = false;
      bool ok = true;
      for (int j0 = 0; j0 < myunits && ok; j0 += kSSets)
        for (int c = 0; c < nchunks && ok; ++c)
          for (int set = 0; set < kSSets && ok; ++set) {
            const int j = j0 + set;
            if (j >= myunits) break;
            const int u = nunits - 1 - static_cast<int>(blockIdx.x + j * gridDim.x);
            const int m = u / HS, hs = u - m * HS;
            const int xq = (hs >> 1) * dq + (hs & 1) * half;
            for (int kb = 0; kb < kiters; ++kb) {
              if (!mbar_wait(&empty[s], ph ^ 1, status, abort)) { ok = false; break; }
              uint8_t* a = stages + s * kSStageBytes;
              mbar_arrive_expect_tx(&full[s], kSStageBytes);
#pragma unroll
              for (int p = 0; p < kScorePlanes; ++p)
                tma_load_3d(a + p * kSPlaneBytes, &tm_planes, &full[s], xq + kb * kSK,
                            m * kRowsPerTile, p);
              tma_load_2d(a + kSABytes, &tm_keys, &full[s], kb * kSK, hs * n + c * kColsPerMma);
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
                   global_timer_ns() - t0 < kDrainLimitNs) {
            }
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer: chunk of 256 sub-keys = kiters x planes x 2 MMAs
      const uint32_t idesc = idesc_bf16_f32(kRowsPerTile, kColsPerMma);
      uint32_t s = 0, ph = 0;
      int uses[kSSets] = {};  // chunks written into each set's accumulators so far
      bool ok = true;
      for (int j0 = 0; j0 < myunits && ok; j0 += kSSets)
        for (int c = 0; c < nchunks && ok; ++c)
          for (int set = 0; set < kSSets && ok; ++set) {
            if (j0 + set >= myunits) break;
            // Set `set` owns accumulator `set`; its uses alternate the barrier phase.
            const int b = set;
            const uint32_t tph = uses[set] & 1;
            if (!mbar_wait(&tempty[b], tph ^ 1, status, abort)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + b * kColsPerMma;
            for (int kb = 0; kb < kiters; ++kb) {
              if (!mbar_wait(&full[s], ph, status, abort)) { ok = false; break; }
              tc_fence_after();
              const uint32_t a = smem_addr(stages + s * kSStageBytes);
              const uint32_t bb = a + kSABytes;
#pragma unroll
              for (int p = 0; p < kScorePlanes; ++p)
#pragma unroll
                for (int jj = 0; jj < kSK / 16; ++jj)
                  mma_bf16(d_tmem, sw64_desc(a + p * kSPlaneBytes, jj * 32), sw64_desc(bb, jj * 32),
                           idesc, (kb | p | jj) != 0);
              mma_commit(&empty[s]);
              if (++s == kSStages) { s = 0; ph ^= 1; }
            }
            if (ok) mma_commit(&tfull[b]);
            ++uses[set];
          }
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kDrainLimitNs) {
      }
    }
  } else {
    // ---------------- epilogue: the best 32 of each row (= TMEM lane)
    // Ls holds the 32 largest scores seen so far (values only, sorted); the log in
    // shared memory holds (score, id) of every element that can still be among the
    // best 32. Columns arrive in increasing sub-key id, so the log is in id order.
    // A chunk is read 8 columns per step with the next step's TMEM load in flight, and
    // the accumulator goes back to the MMA issuer as soon as its last columns are read:
    // the merge that normally follows a chunk runs after that, while the MMAs of the
    // set's next chunk proceed.
    const int set = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    float* lg_s = lg_s_all + set * kSLogRows * kRowsPerTile;  // [kSLogRows][128]
    uint16_t* lg_i = lg_i_all + set * kSLogRows * kRowsPerTile;
    // Shared-window addresses of this row's log column: entry e of the row is at
    // s_row + e * kSStrideS (score) and i_row + e * kSStrideI (id).
    constexpr uint32_t kSStrideS = kRowsPerTile * 4, kSStrideI = kRowsPerTile * 2;
    const uint32_t s_row = smem_addr(lg_s + r), i_row = smem_addr(lg_i + r);
    const uint32_t acc0 = tmem_base + lane_addr + set * kColsPerMma;  // this set's accumulator
    int uses = 0;
    for (int j = set; j < myunits; j += kSSets) {
      const int u = nunits - 1 - static_cast<int>(blockIdx.x + j * gridDim.x);
      const int m = u / HS, hs = u - m * HS;
      float Ls[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) Ls[i] = -INFINITY;
      // A score can still be among the best 32 only if it is >= tau0 (a lower bound of
      // the 32nd best of the first chunk, hence of the row) and > tau_run (the current
      // 32nd best: an equal score comes later in id order and loses the tie).
      float tau0 = -INFINITY, tau_run = -INFINITY;
      float thr = -INFINITY;   // v > thr  <=>  v >= tau0 && v > tau_run
      int cnt = 0, kept = 0;   // log entries; entries kept by the last merge
      bool ok = true;

      // Filter of 8 columns: a kept score and its id go to the next free log slot. The
      // stores and the slot advance are predicated on the compare (no branch, so the
      // warp's rows never diverge), and a rejected score costs no shared-memory store
      // (storing every score and advancing only for kept ones measured 5 us slower).
      auto filter = [&](const uint32_t (&rv)[8], int id0) {
        uint32_t as = s_row + cnt * kSStrideS, ai = i_row + cnt * kSStrideI;
#pragma unroll
        for (int i = 0; i < kSStep; ++i) {
          const float v = __uint_as_float(rv[i]);
          if (v > thr) {
            sts_f32(as, v);
            sts_u16(ai, static_cast<uint16_t>(id0 + i));
            as += kSStrideS;
            ai += kSStrideI;
          }
        }
        cnt = static_cast<int>((as - s_row) / kSStrideS);
      };

      // Merge every fresh log entry into Ls (32 at a time; a round in which no row of the
      // warp has more than 16 fresh entries sorts 16) and raise tau_run. Entries
      // below tau_run can stay in the log: it is compacted to the entries that can
      // still be among the best 32 only when it is filling up, and after the unit.
      auto merge = [&](bool last) {
#pragma unroll 1
        for (int base = kept; __any_sync(0xffffffffu, base < cnt); base += 32) {
          const int fresh = cnt - base;
          const uint32_t fresh_at = s_row + base * kSStrideS;
          if (__reduce_max_sync(0xffffffffu, fresh) <= 16) {
            float b[16];
#pragma unroll
            for (int q = 0; q < 16; ++q)
              b[q] = q < fresh ? lds_f32(fresh_at + q * kSStrideS) : -INFINITY;
            thread_sort16f(b);
#pragma unroll
            for (int i = 16; i < 32; ++i) Ls[i] = fmaxf(Ls[i], b[31 - i]);
          } else {
            float b[32];
#pragma unroll
            for (int q = 0; q < 32; ++q)
              b[q] = q < fresh ? lds_f32(fresh_at + q * kSStrideS) : -INFINITY;
            thread_sort32f(b);
#pragma unroll
            for (int i = 0; i < 32; ++i) Ls[i] = fmaxf(Ls[i], b[31 - i]);
          }
#pragma unroll
          for (int stride = 16; stride > 0; stride >>= 1)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int jj = i ^ stride;
              if (jj > i) {
                const float x0 = Ls[i], x1 = Ls[jj];
                Ls[i] = fmaxf(x0, x1);
                Ls[jj] = fminf(x0, x1);
              }
            }
        }
        tau_run = Ls[31];
        thr = fmaxf(nextafterf(tau0, -INFINITY), tau_run);
        if (!__any_sync(0xffffffffu, last || cnt > kSCompactAt)) {
          kept = cnt;
          return;
        }
        // Branch-free in-place compaction to the entries >= tau_run: every entry is
        // written to the current write slot, which only advances for a kept entry (w <= e,
        // so nothing unread is overwritten). That keeps the current best 32 plus any
        // later entry tied with the 32nd score.
        const int cmax = __reduce_max_sync(0xffffffffu, cnt);
        uint32_t ws = s_row, wi = i_row;
#pragma unroll 4
        for (int e = 0; e < cmax; ++e) {
          const float sv = lds_f32(s_row + e * kSStrideS);
          const uint16_t iv = lds_u16(i_row + e * kSStrideI);
          sts_f32(ws, sv);
          sts_u16(wi, iv);
          if (e < cnt && sv >= tau_run) {
            ws += kSStrideS;
            wi += kSStrideI;
          }
        }
        int w = static_cast<int>((ws - s_row) / kSStrideS);
        if (__any_sync(0xffffffffu, w > kList)) {
          // Rare: ties at the 32nd score. Of the entries equal to tau_run keep the first
          // `eq` in id order (eq = how many of the best 32 scores equal it), so the log
          // is exactly the best 32 by (score desc, id asc).
          int eq = 0;
#pragma unroll
          for (int i = 0; i < 32; ++i) eq += Ls[i] == tau_run ? 1 : 0;
          const int wmax = __reduce_max_sync(0xffffffffu, w);
          int w2 = 0;
          for (int e = 0; e < wmax; ++e) {
            const float sv = lg_s[e * kRowsPerTile + r];
            const uint16_t iv = lg_i[e * kRowsPerTile + r];
            const bool tie = e < w && sv == tau_run && eq > 0;
            const bool keep = e < w && (sv > tau_run || tie);
            eq -= tie ? 1 : 0;
            const int dst = keep ? w2 : kSTrash;
            lg_s[dst * kRowsPerTile + r] = sv;
            lg_i[dst * kRowsPerTile + r] = iv;
            w2 += keep ? 1 : 0;
          }
          w = w2;
        }
        cnt = w;
        kept = w;
      };

#pragma unroll 1
      for (int c = 0; c < nchunks; ++c) {
        if (!warp_wait(&tfull[set], (uses + c) & 1, status, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (c == 0) {
          // The maxima of the 64 groups of 4 columns are 64 different scores of the
          // chunk, so its 32nd best (and the row's) is at least the 32nd largest.
          float mx[64];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            float w[32];
            tmem_ld32(acc0 + g * 32, w);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              mx[g * 8 + i] = fmaxf(fmaxf(w[4 * i], w[4 * i + 1]), fmaxf(w[4 * i + 2], w[4 * i + 3]));
          }
          tau0 = kth32_of_64(mx);
          thr = fmaxf(nextafterf(tau0, -INFINITY), tau_run);
        }
        const int id_base = c * kColsPerMma;
        const bool last_chunk = c == nchunks - 1;
        uint32_t ra[8], rb[8];
        tmem_ld8_issue(acc0, ra);
#pragma unroll 1
        for (int st = 0; st < kSSteps; st += 2) {
          tmem_wait_ld8(ra);
          tmem_ld8_issue(acc0 + (st + 1) * kSStep, rb);
          filter(ra, id_base + st * kSStep);
          tmem_wait_ld8(rb);
          const bool chunk_end = st + 2 >= kSSteps;
          if (!chunk_end) {
            tmem_ld8_issue(acc0 + (st + 2) * kSStep, ra);
          } else {
            // Every column of the accumulator has been read: hand it back.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[set]);
          }
          filter(rb, id_base + (st + 1) * kSStep);
          // Merge when enough is fresh or the next two steps could overflow the log, after
          // a chunk when enough is fresh, and after the unit's last chunk always.
          const int fresh = cnt - kept;
          const int limit = !chunk_end ? kSMidMerge : kSEndMerge;
          const bool unit_end = chunk_end && last_chunk;
          if (__any_sync(0xffffffffu, unit_end || fresh > limit || cnt > kSFull)) merge(unit_end);
        }
      }
      uses += nchunks;
      if (!ok) break;
      const int64_t row = static_cast<int64_t>(m) * kRowsPerTile + r;
      if (row < B) {
        // The log now holds exactly the best 32 (in id order); the candidate kernel
        // sorts them.
        const int64_t o = (row * HS + hs) * static_cast<int64_t>(kList);
#pragma unroll 4
        for (int q = 0; q < kList; ++q) {
          const bool have = q < cnt;
          list_s[o + q] = have ? lg_s[q * kRowsPerTile + r] : -INFINITY;
          list_i[o + q] = have ? static_cast<int>(lg_i[q * kRowsPerTile + r]) : kIdPad;
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

}  // namespace

// bf16 tensor map with a {64 x rows} box and the 128-byte swizzle. dims/strides are
// innermost first; strides are in bytes for dims 1.. (dim 0 is contiguous).
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  const int nplanes = a.raw_acc ? 3 : kScorePlanes;
  CUtensorMap tm_x, tm_w;
  const cuuint64_t xd[2] = {static_cast<cuuint64_t>(a.d_model), static_cast<cuuint64_t>(a.B)};
  const cuuint64_t xs[1] = {static_cast<cuuint64_t>(a.d_model) * 2};
  const cuuint32_t xb[2] = {kKBlock, kRowsPerTile};
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(a.d_model), static_cast<cuuint64_t>(F)};
  const cuuint32_t wb[2] = {kKBlock, kColsPerMma};
  CUtensorMap tm_out;
  const cuuint64_t od[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(a.B),
                            static_cast<cuuint64_t>(nplanes)};
  const cuuint64_t os[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(F) * 2 * a.B};
  const cuuint32_t ob[3] = {32, 32, 1};
  if (!make_map(&tm_x, a.x, 2, xd, xs, xb) || !make_map(&tm_w, a.W_q, 2, wd, xs, wb) ||
      !make_map(&tm_out, planes, 3, od, os, ob, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  const int64_t tiles = ((a.B + kRowsPerTile - 1) / kRowsPerTile) * (F / kColsPerMma);
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  static_assert(kScorePlanes == 2, "the forward's query kernel writes two planes");
  if (nplanes == 2) {
    const size_t smem = query_tc_smem_bytes<2>();
    cudaError_t e = set_max_smem(reinterpret_cast<const void*>(query_tc_kernel<2>), smem);
    if (e != cudaSuccess) return e;
    query_tc_kernel<2><<<grid, kTcThreads, smem, st>>>(tm_x, tm_w, tm_out, a.bn_mean, a.bn_var,
                                                       a.bn_gamma, a.bn_beta, a.bn_eps,
                                                       static_cast<int>(a.B), a.d_model, F,
                                                       a.raw_acc, a.status);
  } else {
    const size_t smem = query_tc_smem_bytes<3>();
    cudaError_t e = set_max_smem(reinterpret_cast<const void*>(query_tc_kernel<3>), smem);
    if (e != cudaSuccess) return e;
    query_tc_kernel<3><<<grid, kTcThreads, smem, st>>>(tm_x, tm_w, tm_out, a.bn_mean, a.bn_var,
                                                       a.bn_gamma, a.bn_beta, a.bn_eps,
                                                       static_cast<int>(a.B), a.d_model, F,
                                                       a.raw_acc, a.status);
  }
  return cudaGetLastError();
}

cudaError_t launch_score_topk_tc(const LayerArgs& a, const void* planes, float* list_s,
                                 int* list_i, cudaStream_t st) {
  const int F = a.H * a.dq;
  const int half = a.dq / 2;
  CUtensorMap tm_p, tm_k;
  const cuuint64_t pd[3] = {static_cast<cuuint64_t>(F), static_cast<cuuint64_t>(a.B),
                            static_cast<cuuint64_t>(kScorePlanes)};
  const cuuint64_t ps[2] = {static_cast<cuuint64_t>(F) * 2, static_cast<cuuint64_t>(F) * 2 * a.B};
  const cuuint32_t pb[3] = {kSK, kRowsPerTile, 1};
  const cuuint64_t kd[2] = {static_cast<cuuint64_t>(half),
                            static_cast<cuuint64_t>(a.H) * 2 * a.n};
  const cuuint64_t ks[1] = {static_cast<cuuint64_t>(half) * 2};
  const cuuint32_t kbx[2] = {kSK, kColsPerMma};
  if (!make_map(&tm_p, planes, 3, pd, ps, pb, kSSwizzle) ||
      !make_map(&tm_k, a.subkeys, 2, kd, ks, kbx, kSSwizzle))
    return cudaErrorInvalidValue;
  const size_t smem = score_tc_smem_bytes();
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(score_topk_tc_kernel), smem);
  if (e != cudaSuccess) return e;
  const int64_t units = ((a.B + kRowsPerTile - 1) / kRowsPerTile) * 2 * a.H;
  const int grid = static_cast<int>(units < sm_count() ? units : sm_count());
  score_topk_tc_kernel<<<grid, kSThreads, smem, st>>>(tm_p, tm_k, static_cast<int>(a.B), a.H,
                                                      a.dq, a.n, list_s, list_i, a.status);
  return cudaGetLastError();
}

}  // namespace pkm
