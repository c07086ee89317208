// pkm_backward.cu -- sparse value backward of the PKM layer.
//
// "Large Memory Layers with Product Keys" (gptget.net summary, Methodology: the
// layer is trained end-to-end with sparse updates; Deep Analysis / Methodology:
// every parameter learns by backpropagation while only a few memory slots are
// updated). With L = <grad_out, out> and out = sum_h sum_j w_j V[slot_j]:
//   grad wrt kept score j:  w_j (g_j - sum_l w_l g_l),  g_j = <grad_out[t], V[slot_j]>
//   grad wrt V[slot]:       sum over the picks of that slot of w * grad_out[t]
//
// The value gradient is deterministic and uses no atomics on rows:
//   1. a stable LSD radix sort (11-bit digits, two passes up to 2^22 slots) groups
//      the B*H*k picks by slot
//      and keeps each slot's picks in pick order;
//   2. one warp per window of 32 sorted picks takes every group that starts in its
//      window: a group of at most kSmallGroup picks is summed in pick order in
//      registers and its row is read and written once;
//   3. a larger group becomes work items of at most kChunk picks: one block per item,
//      eight warps on eight consecutive slices, their sums added in warp order;
//   4. a group of more than kChunk picks writes one partial row per item, and one
//      block per such group adds them in item order before its read-modify-write.
// So every row's sum has the same order on every run, and hot slots are spread over
// many blocks instead of serialising on one row.
#include "pkm_common.cuh"
#include "pkm_kernels.h"

namespace pkm {

constexpr int kScanPer = 4;
constexpr int kScanThreads = 1024;
constexpr int kScanBlock = kScanPer * kScanThreads;  // counts per scan block

static int64_t scan_blocks(int64_t slots) { return (slots + kScanBlock - 1) / kScanBlock; }

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Radix sort geometry: each block of a pass owns kSortTile consecutive positions,
// ranked in sub-tiles of kSortSub (eight warps x 16 steps of 32 keys).
constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortSteps = 16;
constexpr int kSortPerWarp = kSortSteps * 32;
constexpr int kSortSub = kSortWarps * kSortPerWarp;     // 4096
constexpr int kSortSubTiles = 1;
constexpr int kSortTile = kSortSub * kSortSubTiles;     // 4096
constexpr int kDigitBits = 11;
constexpr int kDigits = 1 << kDigitBits;                // 2048
constexpr int kDigitsPerThread = kDigits / kSortThreads;  // 8
static_assert(kDigits % kSortThreads == 0, "digits split evenly over the threads");

// Group sizes: up to kSmallGroup picks a warp sums inline; larger groups are cut into
// work items of at most kChunk picks, one block each.
constexpr int kSmallGroup = kValueSmallGroup;
constexpr int kChunk = kValueChunk;
constexpr int kItemWarps = 8;
static_assert(kSortTile == kSortTileKeys, "tile size shared with the workspace bound");

static int64_t sort_blocks(int64_t E) { return (E + kSortTile - 1) / kSortTile; }

// Radix passes for keys in [0, slots] (slots itself marks an id outside the table).
static int sort_passes(int64_t slots) {
  int bits = 0;
  while (bits < 62 && (static_cast<int64_t>(1) << bits) <= slots) ++bits;
  return (bits + kDigitBits - 1) / kDigitBits;
}

int backward_values_launches(int64_t slots, bool grad_scores, bool grad_values) {
  return (grad_scores ? 1 : 0) + (grad_values ? 3 * sort_passes(slots) + 3 : 0);
}

size_t backward_ws_bytes(int64_t B, int H, int k, int64_t slots, int v, BackwardWs* carve,
                         char* base) {
  const int64_t E = B * H * k;
  const int64_t E1 = E > 0 ? E : 1;
  const int64_t nblk = sort_blocks(E1);
  // Hard bounds of the work lists: a group of more than kSmallGroup picks makes one
  // item per kChunk picks, at most two per kChunk picks when it has more than kChunk.
  const int64_t max_items = value_bwd_max_items(E);
  const int64_t max_huge = value_bwd_max_huge(E);
  const int64_t max_chunks = value_bwd_max_chunks(E);
  size_t off = kStatusBytes;
  const size_t o_ctr = off;      off += 8448;  // list lengths [4], digit totals [64, 2112)
  const size_t o_k0 = off;       off += align256(sizeof(int) * E1);
  const size_t o_p0 = off;       off += align256(sizeof(int) * E1);
  const size_t o_k1 = off;       off += align256(sizeof(int) * E1);
  const size_t o_p1 = off;       off += align256(sizeof(int) * E1);
  const size_t o_hist = off;     off += align256(sizeof(int) * kDigits * nblk);
  const size_t o_items = off;    off += align256(sizeof(int4) * max_items);
  const size_t o_huge = off;     off += align256(sizeof(int4) * max_huge);
  const size_t o_scr = off;      off += align256(sizeof(float) * max_chunks * (v > 0 ? v : 1));
  if (carve && base) {
    carve->ctr = reinterpret_cast<int*>(base + o_ctr);
    carve->keys[0] = reinterpret_cast<int*>(base + o_k0);
    carve->picks[0] = reinterpret_cast<int*>(base + o_p0);
    carve->keys[1] = reinterpret_cast<int*>(base + o_k1);
    carve->picks[1] = reinterpret_cast<int*>(base + o_p1);
    carve->hist = reinterpret_cast<int*>(base + o_hist);
    carve->items = reinterpret_cast<int4*>(base + o_items);
    carve->huge = reinterpret_cast<int4*>(base + o_huge);
    carve->scratch = reinterpret_cast<float*>(base + o_scr);
    carve->max_items = max_items;
    carve->max_huge = max_huge;
    carve->max_chunks = max_chunks;
  }
  (void)slots;
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

// ------------------------------------------- counting sort (full backward's sub-keys)
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

// ------------------------------------------------------- stable LSD radix sort
// Pass `first` reads the slot ids themselves (position p holds pick p); an id outside
// [0, slots) sorts last under the key `slots` (recorded in the status word once per id
// by the histogram pass). Later passes read the previous pass's (key, pick) pairs.
__device__ __forceinline__ int sort_key(const int* keys, int64_t p, int64_t slots, int first) {
  const int k = keys[p];
  return (first && (k < 0 || k >= slots)) ? static_cast<int>(slots) : k;
}

// Digit counts of one tile, written digit-major: hist[d * nblk + block]. Each thread
// loads its kSortSteps keys before counting; a warp adds each distinct digit of a step
// once (the lanes sharing it found by __match_any_sync).
__global__ void __launch_bounds__(kSortThreads) radix_hist_kernel(
    const int* __restrict__ keys, int64_t E, int64_t slots, int shift, int first,
    int* __restrict__ hist, int64_t nblk, int* status) {
  __shared__ int h[kDigits];
#pragma unroll
  for (int i = 0; i < kDigitsPerThread; ++i) h[threadIdx.x + i * kSortThreads] = 0;
  const int lane = threadIdx.x & 31;
  const unsigned lower = (1u << lane) - 1u;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSortTile;
  int raw[kSortSteps];
#pragma unroll
  for (int r = 0; r < kSortSteps; ++r) {
    const int64_t p = base + r * kSortThreads + threadIdx.x;
    raw[r] = p < E ? keys[p] : 0;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortSteps; ++r) {
    const int64_t p = base + r * kSortThreads + threadIdx.x;
    const bool valid = p < E;
    int key = raw[r];
    if (first && valid && (key < 0 || key >= slots)) {
      record_status(status, kDevBadSlot);
      key = static_cast<int>(slots);
    }
    const int d = valid ? (key >> shift) & (kDigits - 1) : kDigits;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    if (valid && (peers & lower) == 0) atomicAdd(&h[d], __popc(peers));  // a count: any order
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kDigitsPerThread; ++i) {
    const int d = threadIdx.x + i * kSortThreads;
    hist[d * nblk + blockIdx.x] = h[d];
  }
}

// Per digit, the exclusive scan of its counts over the blocks, in place (one warp per
// digit, the row read 32 counts at a time), and the digit's total.
__global__ void __launch_bounds__(256) radix_scan_kernel(int* __restrict__ hist, int64_t nblk,
                                                        int* __restrict__ totals) {
  const int lane = threadIdx.x & 31;
  const int d = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (d >= kDigits) return;
  int* row = hist + static_cast<int64_t>(d) * nblk;
  int run = 0;
  for (int64_t b0 = 0; b0 < nblk; b0 += 32) {
    const int64_t b = b0 + lane;
    const int c = b < nblk ? row[b] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (b < nblk) row[b] = run + incl - c;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) totals[d] = run;
}

// Stable scatter of one tile: a key's new position is its digit's offset for this
// block (the scan) + the keys of that digit before it in the tile. Ranks inside a
// warp step come from __match_any_sync (lanes in order), steps and warps follow in
// position order, so equal digits keep their order.
__global__ void __launch_bounds__(kSortThreads) radix_scatter_kernel(
    const int* __restrict__ keys_in, const int* __restrict__ picks_in, int64_t E,
    int64_t slots, int shift, int first, const int* __restrict__ hist, int64_t nblk,
    const int* __restrict__ totals, int* __restrict__ keys_out, int* __restrict__ picks_out) {
  extern __shared__ int sc_smem[];
  int (*cnt)[kDigits] = reinterpret_cast<int (*)[kDigits]>(sc_smem);  // [kSortWarps][kDigits]
  int* base = sc_smem + kSortWarps * kDigits;                         // [kDigits]
  __shared__ int warp_tot[kSortWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lower = (1u << lane) - 1u;
  {
    // Digit d starts after every smaller digit's keys (the exclusive scan of the
    // totals; thread t holds digits [8t, 8t + 8)) and this digit's keys in earlier
    // blocks.
    const int d0 = threadIdx.x * kDigitsPerThread;
    int t[kDigitsPerThread];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kDigitsPerThread; ++i) {
      t[i] = totals[d0 + i];
      sum += t[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int run = incl - sum;
    for (int w = 0; w < warp; ++w) run += warp_tot[w];
#pragma unroll
    for (int i = 0; i < kDigitsPerThread; ++i) {
      base[d0 + i] = run + hist[static_cast<int64_t>(d0 + i) * nblk + blockIdx.x];
      run += t[i];
    }
  }
  for (int sub = 0; sub < kSortSubTiles; ++sub) {
    for (int d = lane; d < kDigits; d += 32) cnt[warp][d] = 0;
    __syncthreads();  // base complete, counters zeroed
    const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kSortTile +
                       static_cast<int64_t>(sub) * kSortSub + warp * kSortPerWarp;
    int key[kSortSteps], pick[kSortSteps], rank[kSortSteps];
#pragma unroll
    for (int r = 0; r < kSortSteps; ++r) {
      const int64_t p = p0 + r * 32 + lane;
      const bool valid = p < E;
      key[r] = valid ? sort_key(keys_in, p, slots, first) : 0;
      pick[r] = valid ? (picks_in ? picks_in[p] : static_cast<int>(p)) : 0;
      const int d = valid ? (key[r] >> shift) & (kDigits - 1) : kDigits;
      const unsigned peers = __match_any_sync(0xffffffffu, d);
      const int before = __popc(peers & lower);
      rank[r] = valid ? cnt[warp][d] + before : 0;
      __syncwarp();
      if (valid && before == 0) cnt[warp][d] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kDigitsPerThread; ++i) {
      // Digit d's positions for this sub-tile: the block's earlier keys, then the
      // warps in order.
      const int d = threadIdx.x + i * kSortThreads;
      int run = base[d];
#pragma unroll
      for (int w = 0; w < kSortWarps; ++w) {
        const int c = cnt[w][d];
        cnt[w][d] = run;
        run += c;
      }
      base[d] = run;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSortSteps; ++r) {
      const int64_t p = p0 + r * 32 + lane;
      if (p < E) {
        const int pos = cnt[warp][(key[r] >> shift) & (kDigits - 1)] + rank[r];
        keys_out[pos] = key[r];
        picks_out[pos] = pick[r];
      }
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------- segmented row sums
// Position just past the group of key r that contains position s (keys sorted
// ascending): the first position q > s with key != r, or E. The warp probes 32
// positions at once, first at distances 1, 2, 4, ... from s, then evenly inside the
// bracket that holds the end (about 32x narrower per round).
__device__ int64_t group_end(const int* __restrict__ skey, int64_t E, int64_t s, int r) {
  const int lane = threadIdx.x & 31;
  int64_t q = s + (static_cast<int64_t>(1) << lane);
  if (q > E) q = E;
  bool past = q >= E || skey[q] != r;
  unsigned b = __ballot_sync(0xffffffffu, past);   // lane 31 reaches E: never empty
  int j = __ffs(b) - 1;
  int64_t hi = __shfl_sync(0xffffffffu, q, j);
  const int64_t qp = __shfl_sync(0xffffffffu, q, j > 0 ? j - 1 : 0);
  int64_t lo = j == 0 ? s + 1 : qp + 1;
  // Invariant: the key at lo - 1 is r, and hi is E or holds another key.
  while (lo < hi) {
    const int64_t span = hi - lo;
    q = lo + span * lane / 32;
    past = skey[q] != r;
    b = __ballot_sync(0xffffffffu, past);
    if (b == 0) {
      lo = lo + span * 31 / 32 + 1;
    } else {
      j = __ffs(b) - 1;
      const int64_t qj = __shfl_sync(0xffffffffu, q, j);
      const int64_t qb = __shfl_sync(0xffffffffu, q, j > 0 ? j - 1 : 0);
      hi = qj;
      if (j > 0) lo = qb + 1;
    }
  }
  return hi;
}

// acc += sum over the sorted positions [a, b) in order of w[pick] * grad_out[token];
// each lane holds the vectors lane, lane + 32, ... of the row.
template <typename T, int MAXV>
__device__ __forceinline__ void sum_picks(const int* __restrict__ spick, int64_t a, int64_t b,
                                          const float* __restrict__ weights,
                                          const T* __restrict__ grad_out, int HK, int v,
                                          float (&acc)[MAXV][Vec<T>::kPer]) {
  constexpr int VPER = Vec<T>::kPer;
  const int lane = threadIdx.x & 31;
  const int nvec = v / VPER;
  for (int64_t c0 = a; c0 < b; c0 += 32) {
    int e_l = 0;
    float w_l = 0.f;
    if (c0 + lane < b) {
      e_l = spick[c0 + lane];
      w_l = weights[e_l];
    }
    const int nb = static_cast<int>(b - c0 < 32 ? b - c0 : 32);
    int j = 0;
    for (; j + 1 < nb; j += 2) {  // two picks in flight
      const int ea = __shfl_sync(0xffffffffu, e_l, j);
      const int eb = __shfl_sync(0xffffffffu, e_l, j + 1);
      const float wa = __shfl_sync(0xffffffffu, w_l, j);
      const float wb = __shfl_sync(0xffffffffu, w_l, j + 1);
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
    if (j < nb) {
      const int ea = __shfl_sync(0xffffffffu, e_l, j);
      const float wa = __shfl_sync(0xffffffffu, w_l, j);
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
  }
}

// acc += the picks at window lanes [j0, j1) in order, each lane l holding pick e_l with
// weight w_l (the window's own loads, handed out by shuffles).
template <typename T, int MAXV>
__device__ __forceinline__ void sum_window_picks(int e_l, float w_l, int j0, int j1,
                                                 const T* __restrict__ grad_out, int HK, int v,
                                                 float (&acc)[MAXV][Vec<T>::kPer]) {
  constexpr int VPER = Vec<T>::kPer;
  const int lane = threadIdx.x & 31;
  const int nvec = v / VPER;
  int j = j0;
  for (; j + 1 < j1; j += 2) {  // two picks in flight
    const int ea = __shfl_sync(0xffffffffu, e_l, j);
    const int eb = __shfl_sync(0xffffffffu, e_l, j + 1);
    const float wa = __shfl_sync(0xffffffffu, w_l, j);
    const float wb = __shfl_sync(0xffffffffu, w_l, j + 1);
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
  if (j < j1) {
    const int ea = __shfl_sync(0xffffffffu, e_l, j);
    const float wa = __shfl_sync(0xffffffffu, w_l, j);
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
}

// One warp per window of 32 sorted picks; the warp takes every group that starts in
// its window. Groups of at most kSmallGroup picks: summed here and the row written
// once (the only writer of that row). Larger groups: appended to the work lists.
template <typename T, int MAXV>
__global__ void __launch_bounds__(128) segment_small_kernel(
    const int* __restrict__ skey, const int* __restrict__ spick, int64_t E, int64_t slots,
    const float* __restrict__ weights, const T* __restrict__ grad_out, int HK, int v,
    float* __restrict__ grad_values, int* __restrict__ ctr, int4* __restrict__ items,
    int4* __restrict__ huge) {
  constexpr int VPER = Vec<T>::kPer;
  const int lane = threadIdx.x & 31;
  const int nvec = v / VPER;
  const int end_key = static_cast<int>(slots);  // past the table: never a group
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t win = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       win * 32 < E; win += nwarps) {
    const int64_t w0 = win * 32;
    // Keys, picks and weights of this window and of the next one, loaded together:
    // groups that start here and end within the next window need no further loads.
    const int key = w0 + lane < E ? skey[w0 + lane] : end_key;
    const int key_b = w0 + 32 + lane < E ? skey[w0 + 32 + lane] : end_key;
    int e_l = 0, e_b = 0;
    float w_l = 0.f, w_b = 0.f;
    if (key < end_key) {
      e_l = spick[w0 + lane];
      w_l = weights[e_l];
    }
    if (key_b < end_key) {
      e_b = spick[w0 + 32 + lane];
      w_b = weights[e_b];
    }
    int prev = __shfl_up_sync(0xffffffffu, key, 1);
    if (lane == 0) prev = w0 > 0 ? skey[w0 - 1] : -1;
    unsigned starts = __ballot_sync(0xffffffffu, key < end_key && key != prev);
    while (starts) {
      const int s = __ffs(starts) - 1;
      starts &= starts - 1;
      const int r = __shfl_sync(0xffffffffu, key, s);
      const unsigned change = __ballot_sync(0xffffffffu, lane > s && key != r);
      const unsigned change_b = __ballot_sync(0xffffffffu, key_b != r);
      const int64_t g0 = w0 + s;
      const int64_t g1 = change     ? w0 + __ffs(change) - 1
                         : change_b ? w0 + 32 + __ffs(change_b) - 1
                                    : group_end(skey, E, w0 + 63, r);
      const int64_t size = g1 - g0;
      if (size <= kSmallGroup) {
        float* grow = grad_values + static_cast<int64_t>(r) * v;
        float4 old[MAXV][VPER / 4];
        float acc[MAXV][VPER];
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          const int vec = lane + 32 * m;
#pragma unroll
          for (int q = 0; q < VPER; q += 4) {
            old[m][q / 4] = vec < nvec ? *reinterpret_cast<const float4*>(grow + vec * VPER + q)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
            acc[m][q] = acc[m][q + 1] = acc[m][q + 2] = acc[m][q + 3] = 0.f;
          }
        }
        // In pick order: this window's lanes, the next window's lanes, then the rest.
        const int in_a = static_cast<int>((g1 < w0 + 32 ? g1 : w0 + 32) - w0);
        sum_window_picks<T, MAXV>(e_l, w_l, s, in_a, grad_out, HK, v, acc);
        if (g1 > w0 + 32) {
          const int in_b = static_cast<int>((g1 < w0 + 64 ? g1 : w0 + 64) - (w0 + 32));
          sum_window_picks<T, MAXV>(e_b, w_b, 0, in_b, grad_out, HK, v, acc);
        }
        if (g1 > w0 + 64) sum_picks<T, MAXV>(spick, w0 + 64, g1, weights, grad_out, HK, v, acc);
#pragma unroll
        for (int m = 0; m < MAXV; ++m) {
          const int vec = lane + 32 * m;
          if (vec < nvec) {
#pragma unroll
            for (int q = 0; q < VPER; q += 4) {
              const float4 o = old[m][q / 4];
              *reinterpret_cast<float4*>(grow + vec * VPER + q) =
                  make_float4(o.x + acc[m][q], o.y + acc[m][q + 1], o.z + acc[m][q + 2],
                              o.w + acc[m][q + 3]);
            }
          }
        }
      } else if (size <= kChunk) {
        if (lane == 0) items[atomicAdd(&ctr[0], 1)] = make_int4(static_cast<int>(g0),
                                                                static_cast<int>(size), r, -1);
      } else {
        // One item per kChunk picks, each writing a partial row; the group's own entry
        // in `huge` lists the partial rows in item order.
        const int nch = static_cast<int>((size + kChunk - 1) / kChunk);
        int i0 = 0, c0 = 0;
        if (lane == 0) {
          i0 = atomicAdd(&ctr[0], nch);
          c0 = atomicAdd(&ctr[2], nch);
          huge[atomicAdd(&ctr[1], 1)] = make_int4(r, c0, nch, 0);
        }
        i0 = __shfl_sync(0xffffffffu, i0, 0);
        c0 = __shfl_sync(0xffffffffu, c0, 0);
        for (int c = lane; c < nch; c += 32) {
          const int64_t a = g0 + static_cast<int64_t>(c) * kChunk;
          const int64_t n = size - static_cast<int64_t>(c) * kChunk;
          items[i0 + c] = make_int4(static_cast<int>(a), static_cast<int>(n < kChunk ? n : kChunk),
                                    r, c0 + c);
        }
      }
    }
  }
}

// One block per work item {start, picks, slot, dest}: eight warps sum eight
// consecutive slices in pick order, then the slices are added in warp order. dest < 0:
// the row is read and written once; else the sum is partial row `dest` of a huge group.
template <typename T, int MAXV>
__global__ void __launch_bounds__(kItemWarps * 32) segment_items_kernel(
    const int* __restrict__ spick, const float* __restrict__ weights,
    const T* __restrict__ grad_out, int HK, int v, const int* __restrict__ ctr,
    const int4* __restrict__ items, float* __restrict__ grad_values,
    float* __restrict__ scratch) {
  constexpr int VPER = Vec<T>::kPer;
  extern __shared__ float4 red4[];  // [kItemWarps][v / 4]
  float* red = reinterpret_cast<float*>(red4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = v / VPER;
  const int nitems = ctr[0];
  for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
    const int4 item = items[it];
    const int per = (item.y + kItemWarps - 1) / kItemWarps;
    const int64_t end = static_cast<int64_t>(item.x) + item.y;
    int64_t a = static_cast<int64_t>(item.x) + static_cast<int64_t>(warp) * per;
    int64_t b = a + per;
    if (a > end) a = end;
    if (b > end) b = end;
    float acc[MAXV][VPER];
#pragma unroll
    for (int m = 0; m < MAXV; ++m)
#pragma unroll
      for (int q = 0; q < VPER; ++q) acc[m][q] = 0.f;
    sum_picks<T, MAXV>(spick, a, b, weights, grad_out, HK, v, acc);
#pragma unroll
    for (int m = 0; m < MAXV; ++m) {
      const int vec = lane + 32 * m;
      if (vec < nvec) {
#pragma unroll
        for (int q = 0; q < VPER; ++q) red[warp * v + vec * VPER + q] = acc[m][q];
      }
    }
    __syncthreads();
    for (int c = threadIdx.x * 4; c < v; c += kItemWarps * 32 * 4) {
      float4 sum = *reinterpret_cast<const float4*>(red + c);
#pragma unroll
      for (int w = 1; w < kItemWarps; ++w) {
        const float4 x = *reinterpret_cast<const float4*>(red + w * v + c);
        sum = make_float4(sum.x + x.x, sum.y + x.y, sum.z + x.z, sum.w + x.w);
      }
      if (item.w < 0) {
        float4* g = reinterpret_cast<float4*>(grad_values + static_cast<int64_t>(item.z) * v + c);
        const float4 o = *g;
        *g = make_float4(o.x + sum.x, o.y + sum.y, o.z + sum.z, o.w + sum.w);
      } else {
        *reinterpret_cast<float4*>(scratch + static_cast<int64_t>(item.w) * v + c) = sum;
      }
    }
    __syncthreads();
  }
}

// One block per group of more than kChunk picks: its partial rows added in item order,
// then one read-modify-write of the row.
__global__ void __launch_bounds__(256) segment_huge_kernel(const int* __restrict__ ctr,
                                                           const int4* __restrict__ huge,
                                                           const float* __restrict__ scratch,
                                                           int v, float* __restrict__ grad_values) {
  const int nh = ctr[1];
  for (int g = blockIdx.x; g < nh; g += gridDim.x) {
    const int4 h = huge[g];
    for (int c = threadIdx.x * 4; c < v; c += 256 * 4) {
      float4 sum = *reinterpret_cast<const float4*>(scratch + static_cast<int64_t>(h.y) * v + c);
      for (int i = 1; i < h.z; ++i) {
        const float4 x =
            *reinterpret_cast<const float4*>(scratch + static_cast<int64_t>(h.y + i) * v + c);
        sum = make_float4(sum.x + x.x, sum.y + x.y, sum.z + x.z, sum.w + x.w);
      }
      float4* gr = reinterpret_cast<float4*>(grad_values + static_cast<int64_t>(h.x) * v + c);
      const float4 o = *gr;
      *gr = make_float4(o.x + sum.x, o.y + sum.y, o.z + sum.z, o.w + sum.w);
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

// Stable sort of the picks by slot; returns which ping-pong buffer holds the result.
constexpr size_t kScatterSmem = sizeof(int) * (kSortWarps + 1) * kDigits;  // 72 KiB

static cudaError_t sort_picks_by_slot(const int* indices, int64_t E, int64_t slots,
                                      const BackwardWs& ws, int* status, cudaStream_t st,
                                      int* which) {
  const int64_t nblk = sort_blocks(E);
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(radix_scatter_kernel), kScatterSmem);
  if (e != cudaSuccess) return e;
  const int passes = sort_passes(slots);
  const int* kin = indices;
  const int* pin = nullptr;
  int cur = 0;
  for (int ps = 0; ps < passes; ++ps) {
    const int shift = kDigitBits * ps;
    const int first = ps == 0;
    radix_hist_kernel<<<static_cast<unsigned>(nblk), kSortThreads, 0, st>>>(
        kin, E, slots, shift, first, ws.hist, nblk, status);
    radix_scan_kernel<<<kDigits / 8, 256, 0, st>>>(ws.hist, nblk, ws.ctr + 64);
    radix_scatter_kernel<<<static_cast<unsigned>(nblk), kSortThreads, kScatterSmem, st>>>(
        kin, pin, E, slots, shift, first, ws.hist, nblk, ws.ctr + 64, ws.keys[cur],
        ws.picks[cur]);
    kin = ws.keys[cur];
    pin = ws.picks[cur];
    cur ^= 1;
  }
  *which = cur ^ 1;
  return cudaGetLastError();
}

// B1: gradients of the kept scores (reads the picked value rows and grad_out).
template <typename T, int MAXV>
static cudaError_t launch_scores_t(int64_t B, int H, int k, int v, int64_t slots,
                                   const void* values, const int* indices, const float* weights,
                                   const void* grad_out, float* grad_scores, int* status,
                                   cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((B + 3) / 4);
  grad_scores_kernel<T, MAXV><<<grid, 128, 0, st>>>(static_cast<const T*>(values),
                                                    static_cast<const T*>(grad_out), indices,
                                                    weights, B, H, k, v, slots, grad_scores,
                                                    status);
  return cudaGetLastError();
}

// B2 in two parts. The sort of the picks by slot (reads only the indices; its keys and
// pick ids stay in L2) ...
static cudaError_t launch_sort_part(int64_t B, int H, int k, int64_t slots, const int* indices,
                                    const BackwardWs& ws, int* status, cudaStream_t st) {
  const int64_t E = B * H * k;
  cudaError_t e = cudaMemsetAsync(ws.ctr, 0, 4 * sizeof(int), st);
  if (e != cudaSuccess) return e;
  int which = 0;
  return sort_picks_by_slot(indices, E, slots, ws, status, st, &which);
}

// ... and each slot's picks summed into its row of grad_values (reads the sorted picks,
// weights and grad_out). Neither part needs B1's result.
template <typename T, int MAXV>
static cudaError_t launch_segments_t(int64_t B, int H, int k, int v, int64_t slots,
                                     const float* weights, const void* grad_out,
                                     float* grad_values, const BackwardWs& ws,
                                     cudaStream_t st) {
  const int64_t E = B * H * k;
  const T* G = static_cast<const T*>(grad_out);
  // sort_picks_by_slot alternates the two buffers, starting with 0.
  const int which = (sort_passes(slots) - 1) & 1;
  const int* skey = ws.keys[which];
  const int* spick = ws.picks[which];
  const int64_t windows = (E + 31) / 32;
  const int64_t sblocks = (windows + 3) / 4;
  const unsigned sgrid = static_cast<unsigned>(sblocks < 148 * 64 ? sblocks : 148 * 64);
  segment_small_kernel<T, MAXV><<<sgrid > 0 ? sgrid : 1, 128, 0, st>>>(
      skey, spick, E, slots, weights, G, H * k, v, grad_values, ws.ctr, ws.items, ws.huge);
  const size_t smem = sizeof(float) * kItemWarps * v;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(segment_items_kernel<T, MAXV>), smem);
  if (e != cudaSuccess) return e;
  segment_items_kernel<T, MAXV><<<2 * 148, kItemWarps * 32, smem, st>>>(
      spick, weights, G, H * k, v, ws.ctr, ws.items, grad_values, ws.scratch);
  segment_huge_kernel<<<148, 256, 0, st>>>(ws.ctr, ws.huge, ws.scratch, v, grad_values);
  return cudaGetLastError();
}

#define PKM_BWD_DISPATCH(FN, ...)                          \
  do {                                                     \
    const int m_ = row_vecs_per_lane(v, dtype);            \
    if (dtype == 0) {                                      \
      switch (m_) {                                        \
        case 1: return FN<float, 1>(__VA_ARGS__);          \
        case 2: return FN<float, 2>(__VA_ARGS__);          \
        case 4: return FN<float, 4>(__VA_ARGS__);          \
        case 8: return FN<float, 8>(__VA_ARGS__);          \
      }                                                    \
    } else {                                               \
      switch (m_) {                                        \
        case 1: return FN<uint16_t, 1>(__VA_ARGS__);       \
        case 2: return FN<uint16_t, 2>(__VA_ARGS__);       \
        case 4: return FN<uint16_t, 4>(__VA_ARGS__);       \
        case 8: return FN<uint16_t, 8>(__VA_ARGS__);       \
      }                                                    \
    }                                                      \
    return cudaErrorInvalidValue;                          \
  } while (0)

cudaError_t launch_grad_scores(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                               const void* values, const int* indices, const float* weights,
                               const void* grad_out, float* grad_scores, int* status,
                               cudaStream_t st) {
  PKM_BWD_DISPATCH(launch_scores_t, B, H, k, v, slots, values, indices, weights, grad_out,
                   grad_scores, status, st);
}

cudaError_t launch_value_sort(int64_t B, int H, int k, int64_t slots, const int* indices,
                              const BackwardWs& ws, int* status, cudaStream_t st) {
  return launch_sort_part(B, H, k, slots, indices, ws, status, st);
}

cudaError_t launch_value_segments(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                                  const float* weights, const void* grad_out, float* grad_values,
                                  const BackwardWs& ws, cudaStream_t st) {
  PKM_BWD_DISPATCH(launch_segments_t, B, H, k, v, slots, weights, grad_out, grad_values, ws, st);
}

cudaError_t launch_value_rows(int64_t B, int H, int k, int v, int dtype, int64_t slots,
                              const int* indices, const float* weights, const void* grad_out,
                              float* grad_values, const BackwardWs& ws, int* status,
                              cudaStream_t st) {
  const cudaError_t e = launch_value_sort(B, H, k, slots, indices, ws, status, st);
  if (e != cudaSuccess) return e;
  return launch_value_segments(B, H, k, v, dtype, slots, weights, grad_out, grad_values, ws, st);
}
#undef PKM_BWD_DISPATCH

}  // namespace pkm
